"""Raw score tiles of the attention kernels against the oracle (GPU, debug capture).

The INT8 path's tile accumulators sum_d cq[i,d] * ck[j,d] (TileMix page, section 2, "The
Dual-Path Engine": quantised Q and K multiplied on the tensor cores, then rescaled) must be
bit-exact.  lamp_attn_debug runs the same kernels and launch configuration as
lamp_attn_fwd_q8 and copies the raw tiles the softmax read out of tensor memory; they are
compared here with ``oracle.score_tiles`` on the GPU's own codes (which the quantiser parity
tests pin to the oracle's):
  * INT8 8-bit tiles: bit-exact (int32);
  * E4M3 8-bit tiles and 16-bit tiles: fp32 accumulation on the tensor core, whose internal
    order and width are not documented, so E4M3 tiles are compared with a tolerance: every product
    is exact in fp32, so the sum of D products is within D * 2^-24 * sum |products| of the
    exact fp64 sum; the test allows 1e-5 * sum |products|;
and, tile by tile, the dump holds a product exactly when the route map says the tile used it
(8-bit: route codes 1, 3; 16-bit: 2, 3).  The capture build must also give O, lse and the
route map bit-identical to the product kernels.
"""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
import oracle
from workloads import CONFIGS, make_workload

from _parity import gpu_mask, to_dev

pytestmark = pytest.mark.gpu

SENT8 = 0x7FBADBAD
REL = 1e-5


def _pick_tiles(route, n, seed):
    """Up to n seeded live tiles, always including each route code present, the last query
    tile and the last key tile (ragged edges)."""
    rng = np.random.default_rng(seed)
    live = np.argwhere(route > 0)
    chosen = {tuple(x) for x in live if x[2] == route.shape[2] - 1 or x[3] == route.shape[3] - 1}
    chosen = set(list(chosen)[: n // 3])
    for code in (1, 2, 3):
        idx = np.argwhere(route == code)
        if len(idx):
            chosen.update(tuple(x) for x in idx[rng.choice(len(idx), min(4, len(idx)), replace=False)])
    rest = live[rng.permutation(len(live))]
    for x in rest:
        if len(chosen) >= n:
            break
        chosen.add(tuple(x))
    return sorted(tuple(int(v) for v in x) for x in chosen)


def _abs_codes(c, fmt):
    """Codes of |value| (INT8: two's complement magnitude; E4M3: sign bit cleared)."""
    if fmt == "int8":
        return np.abs(c.view(np.int8).astype(np.int16)).astype(np.uint8)
    return c & np.uint8(0x7F)


def run_tiles_case(w, *, n_tiles=48, p_fp16=None, route=None, fmt=None, tau=None, seed=0):
    route = route or w.route
    fmt = fmt or w.fmt
    tau = w.tau if tau is None else tau
    t = make_workload(w)
    q, k, v = (to_dev(x, w.dtype) for x in (t.q_bits, t.k_bits, t.v_bits))
    q8, k8, qs, ks = mpt.quantize(q, k, fmt=fmt)
    mask = gpu_mask(w, p_fp16) if route == "bitmask" else None
    kw = dict(causal=w.causal, window=w.window, mask_bits=mask, group_tiles=w.group_tiles,
              route=route, fmt=fmt, tau=tau)
    o_ref, lse_ref, rmap_ref = mpt.attention_q8(q, k, v, q8, k8, qs, ks, want_route=True, **kw)
    torch.cuda.synchronize()
    rmap = rmap_ref.cpu().numpy()
    tiles = _pick_tiles(rmap, n_tiles, seed)
    o, lse, rm, s8, s16 = mpt.attention_debug(q, k, v, q8, k8, qs, ks, tiles, **kw)
    torch.cuda.synchronize()
    mpt.lamp_check()
    # the capture build computes exactly what the product kernel computes
    assert torch.equal(rm, rmap_ref) and torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    qc, kc = q8.cpu().numpy(), k8.cpu().numpy()
    s8n = s8.cpu().numpy()
    s16n = s16.cpu().numpy()
    ex8 = oracle.score_tiles(qc, kc, w.bm, w.bn, fmt, tiles)
    ab8 = oracle.score_tiles(_abs_codes(qc, fmt), _abs_codes(kc, fmt), w.bm, w.bn, fmt, tiles)
    ex16 = oracle.score_tiles(t.q, t.k, w.bm, w.bn, "16bit", tiles)
    ab16 = oracle.score_tiles(np.abs(t.q), np.abs(t.k), w.bm, w.bn, "16bit", tiles)
    seen8 = seen16 = 0
    for s, (b, h, qt, kt) in enumerate(tiles):
        rc = rmap[b, h, qt, kt]
        if rc in (1, 3):
            seen8 += 1
            if fmt == "int8":
                assert np.array_equal(s8n[s].astype(np.int64), ex8[s].astype(np.int64)), \
                    ("int32 tile differs", (b, h, qt, kt), np.argwhere(s8n[s] != ex8[s])[:4])
            else:
                got = s8n[s].view(np.float32).astype(np.float64)
                err = np.abs(got - ex8[s])
                assert np.all(err <= REL * ab8[s] + 1e-30), ("e4m3 tile", (b, h, qt, kt), err.max())
        else:
            assert np.all(s8n[s] == SENT8), ("8-bit dump of a tile without 8-bit pass", rc)
        if rc in (2, 3):
            seen16 += 1
            err = np.abs(s16n[s].astype(np.float64) - ex16[s])
            assert np.all(err <= REL * ab16[s] + 1e-30), ("16-bit tile", (b, h, qt, kt), err.max())
        else:
            assert np.all(np.isnan(s16n[s])), ("16-bit dump of a tile without 16-bit pass", rc)
    return seen8, seen16


TINY = CONFIGS["tiny"]
GQA = CONFIGS["gqa4k"]
GEMMA = CONFIGS["gemma_local16k"]
ADAPT = CONFIGS["adaptive8k"]


def test_tiny_d64_stacked_all_tiles():
    s8, s16 = run_tiles_case(TINY, n_tiles=16)
    assert s8 > 0 and s16 > 0


@pytest.mark.parametrize("p", [0.3, 0.0])
def test_two_tile_kernel_int8_bitmask_small(p):
    w = GQA.replace(B=1, H=4, Hkv=2, Lq=600, Lk=600, group_tiles=1)
    s8, s16 = run_tiles_case(w, n_tiles=100, p_fp16=p)
    assert s8 > 0 and (s16 > 0) == (p > 0)


def test_two_tile_kernel_int8_bitmask_full_size_gqa4k():
    s8, s16 = run_tiles_case(GQA, n_tiles=64, seed=1)
    assert s8 > 0 and s16 > 0


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
@pytest.mark.parametrize("tau", [2.0, -1e30])
def test_look_ahead_tiles_both_kernels(fmt, tau):
    # INT8 runs on the two-tile kernel, E4M3 on the single-tile kernel; a flagged tile has both
    # its 8-bit pass and its 16-bit recomputation captured
    w = ADAPT.replace(B=1, H=4, Hkv=2, Lq=768, Lk=768)
    s8, s16 = run_tiles_case(w, n_tiles=80, fmt=fmt, tau=tau, seed=2)
    assert s8 > 0 and s16 > 0


def test_single_tile_kernel_int8_wide_mask():
    # more than two mask words at D = 128 send INT8 to the single-tile kernel
    w = GQA.replace(B=1, H=2, Hkv=1, Lq=129 * 128, Lk=129 * 128, group_tiles=1, p_fp16=0.5)
    assert mpt.lamp_mask_words(w.Lk, w.D, w.group_tiles) == 3
    s8, s16 = run_tiles_case(w, n_tiles=40, seed=3)
    assert s8 > 0 and s16 > 0


@pytest.mark.parametrize("window", [0, 200])
def test_d256_stacked_halves_mixed_routing(window):
    w = GEMMA.replace(B=1, H=4, Hkv=2, Lq=700, Lk=700, window=window)
    s8, s16 = run_tiles_case(w, n_tiles=80, seed=4)
    assert s8 > 0 and s16 > 0


def test_d256_full_size_gemma_local16k():
    s8, s16 = run_tiles_case(GEMMA, n_tiles=48, seed=5)
    assert s8 > 0 and s16 > 0


@pytest.mark.parametrize("base", ["tiny", "gemma_local16k"])
def test_stacked_look_ahead_tiles(base):
    w = CONFIGS[base].replace(B=1, H=2, Hkv=1, Lq=330, Lk=330, causal=True, route="adaptive",
                              tau=3.0, values="structured", plant_frac=0.02, window=0)
    s8, s16 = run_tiles_case(w, n_tiles=60, fmt="int8", tau=3.0, seed=6)
    assert s8 > 0 and s16 > 0
