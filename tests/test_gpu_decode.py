"""Decode with an 8-bit key/value cache on the GPU (TileMix page, section 4: INT8 key/value
caches for the decode phase), through the C ABI, against the oracle.

Decode is the routed attention of one query row per (batch, head) over the cached keys; the
oracle runs it per sequence with the cache's own 8-bit key codes and scales (k_codes_in), the
dequantised cached keys for the 16-bit route and the dequantised cached values."""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
import oracle
from workloads import CONFIGS, make_workload

from _parity import check_outputs, mask_to_numpy, to_dev

pytestmark = pytest.mark.gpu

E4M3_TABLE = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def dequant(codes, scales, bn, fmt):
    vals = codes.view(np.int8).astype(np.float32) if fmt == "int8" else E4M3_TABLE[codes]
    rep = np.repeat(scales, bn, axis=-1)[..., : codes.shape[-2]]
    return (vals * rep[..., None]).astype(np.float32)


@pytest.mark.parametrize("D,H,Hkv,lens,fmt,p16,g", [
    (128, 8, 2, [1000, 613], "int8", 0.3, 2),
    (64, 4, 2, [300, 0, 129], "e4m3", None, 1),
    (256, 8, 4, [700, 1024], "int8", 0.5, 2),
    (128, 32, 8, [4096], "e4m3", 0.2, 4),
    # long caches: many 128-key chunks and several splits of 8 chunks per CTA, ragged ends
    (128, 32, 8, [20000, 9001], "int8", 0.25, 8),
    (64, 8, 1, [3000, 1025], "e4m3", 0.5, 1),
    (256, 16, 2, [5000], "int8", 0.3, 2),
])
def test_decode_matches_oracle(D, H, Hkv, lens, fmt, p16, g):
    B, max_k = len(lens), max(lens)
    bm, bn = mpt.lamp_tile_shape(D)
    w = CONFIGS["gqa4k"].replace(B=B, H=H, Hkv=Hkv, Lq=1, Lk=max_k, D=D, bm=bm, bn=bn,
                                 group_tiles=g)
    t = make_workload(w)
    q, k, v = (to_dev(x, w.dtype) for x in (t.q_bits, t.k_bits, t.v_bits))
    nkt = -(-max_k // bn)
    mode = mpt.mode_bits("bitmask", fmt, w.dtype)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    qs = torch.empty((B, H, 1), device="cuda")
    k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
    ks = torch.empty((B, Hkv, nkt), device="cuda")
    v8 = torch.empty(v.shape, dtype=torch.uint8, device="cuda")
    vs = torch.empty((B, Hkv, nkt), device="cuda")
    mpt.lamp_quant_qk(q, None, q8, None, qs, None, B, H, Hkv, 1, max_k, D, mode)
    mpt.lamp_quant_qk(None, k, None, k8, None, ks, B, H, Hkv, 1, max_k, D, mode)
    mpt.lamp_quant_qk(None, v, None, v8, None, vs, B, H, Hkv, 1, max_k, D, mode)
    mask = mpt.build_mask(B, H, 1, max_k, D, g, p16, 5) if p16 is not None else None
    len_k = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = torch.full((B, H, D), float("nan"), device="cuda")
    lse = torch.full((B, H), float("nan"), device="cuda")
    mpt.lamp_decode_fwd(q, q8, qs, k8, ks, v8, vs, len_k, o, lse, B, H, Hkv, max_k, D, 0.0, mask,
                        g, mode)
    torch.cuda.synchronize()
    mpt.lamp_check()
    o, lse = o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    k8n, ksn, v8n, vsn = (x.cpu().numpy() for x in (k8, ks, v8, vs))
    mnp = mask_to_numpy(mask) if mask is not None else None
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(o[b] == 0.0) and np.all(np.isneginf(lse[b]))
            continue
        nk = -(-n // bn)
        kc, kcs = k8n[b:b + 1, :, :n], ksn[b:b + 1, :, :nk]
        kv = dequant(kc, kcs, bn, fmt)
        vv = dequant(v8n[b:b + 1, :, :n], vsn[b:b + 1, :, :nk], bn, fmt)
        r = oracle.attention(t.q[b:b + 1], kv, vv, bm=bm, bn=bn, causal=True,
                             mask=None if mnp is None else np.ascontiguousarray(mnp[b:b + 1]),
                             group_tiles=g, fmt=fmt, k_codes_in=kc, k_scales_in=kcs)
        got = {"o": o[b:b + 1, :, None, :], "lse": lse[b:b + 1, :, None]}
        check_outputs(got, r, what=f"decode D={D} {fmt} sequence {b}")
