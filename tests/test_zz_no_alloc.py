"""The allocation-free entry point against the regular one (GPU).

lamp_attn_fwd_noalloc is for callers that cannot allocate device memory: their memory is all
owned by another allocator, or they run latency-bound loops in which cudaMalloc / cudaFree
(which may synchronise the whole device) are not allowed.  Its scratch lives in a fixed device
array inside the library.  This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
from workloads import CONFIGS, make_workload

from _parity import LSE_ABS, O_MAX_ABS, O_MEAN_ABS, to_dev

pytestmark = pytest.mark.gpu


def _run(fn, w, t, mask):
    q, k, v = (to_dev(x, w.dtype) for x in (t.q_bits, t.k_bits, t.v_bits))
    o = torch.empty((w.B, w.H, w.Lq, w.D), device="cuda", dtype=torch.float32)
    lse = torch.empty((w.B, w.H, w.Lq), device="cuda", dtype=torch.float32)
    mode = mpt.mode_bits(w.route, w.fmt, w.dtype)
    fn(q, k, v, o, lse, w.B, w.H, w.Hkv, w.Lq, w.Lk, w.D, int(w.causal), w.window, 0.0, mask,
       w.group_tiles, mode, w.tau)
    torch.cuda.synchronize()
    mpt.lamp_check()
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,kw", [
    ("gqa4k", dict(B=1, H=8, Hkv=2, Lq=1000, Lk=1000)),
    ("tiny", dict(causal=True, values="structured", plant_frac=0.02)),
    ("gemma_local16k", dict(H=2, Hkv=1, Lq=900, Lk=900)),
    ("adaptive8k", dict(B=1, H=4, Hkv=2, Lq=700, Lk=700)),
])
def test_noalloc_matches_regular_entry_point_twice(name, kw):
    w = CONFIGS[name].replace(**kw)
    t = make_workload(w)
    mask = (mpt.build_mask(w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles, w.p_fp16, w.mask_seed)
            if w.route == "bitmask" else None)
    ref_o, ref_lse = _run(mpt.lamp_attn_fwd, w, t, mask)
    fin = np.isfinite(ref_lse)
    # A caller workspace far too small for this problem: if the allocation-free entry point
    # fell through to the workspace path (or to an allocation), the call would fail here.
    tiny = torch.empty(512, dtype=torch.uint8, device="cuda")
    mpt.lamp_set_workspace((tiny.data_ptr() + 255) & ~255, 256)
    try:
        with pytest.raises(mpt.LampError):  # the workspace path does see the small workspace
            _run(mpt.lamp_attn_fwd, w, t, mask)
        for _ in range(2):  # the shared scratch keeps the previous call's contents
            o, lse = _run(mpt.lamp_attn_fwd_noalloc, w, t, mask)
            assert np.array_equal(np.isfinite(lse), fin)
            err = np.abs(o - ref_o)
            assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS
            assert np.abs(lse[fin] - ref_lse[fin]).max() <= LSE_ABS
    finally:
        mpt.lamp_set_workspace(None, 0)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # B*H*Lq*D + B*Hkv*Lk*D bytes of 8-bit operands exceed the fixed array: refused on the host
    B, H, Hkv, L, D = 1, 32, 8, 16384, 128
    assert mpt.lamp_workspace_size(B, H, Hkv, L, L, D) > mpt.NOALLOC_MAX_BYTES
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_attn_fwd_noalloc(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, B, H, Hkv, L, L, D,
                                  1, 0, 0.0, None, 1, mpt.mode_bits(), 0.0)
    assert e.value.code == mpt.LAMP_ERR_INVALID
    assert "scratch" in mpt.lamp_last_error()
