"""Pins of the oracle's raw score tiles and of its hint bookkeeping (CPU).

``oracle.score_tiles`` is the reference of the library's debug capture: the unscaled 8-bit
product sum_d cq[i,d] * ck[j,d] of a routing tile (TileMix page, section 2, "The Dual-Path
Engine": the INT8 path multiplies quantised Q and K on the tensor cores before the rescale), or
the 16-bit product of the inputs.  It is pinned here against computations it does not share:
numpy integer / fp64 matrix products, torch's own e4m3 decoder, a closed form on the zero
padding of ragged tiles, transpose symmetry and the grouped-query head mapping.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_workload


def _codes(rng, shape):
    return rng.integers(0, 256, size=shape).astype(np.uint8)


def _pad_block(x, r0, n, axis_len):
    """Rows [r0, r0 + n) of x [..., L, D], zero past L."""
    out = np.zeros((n, x.shape[-1]), dtype=x.dtype)
    m = max(0, min(n, axis_len - r0))
    out[:m] = x[r0:r0 + m]
    return out


@pytest.mark.parametrize("bm,bn,D", [(64, 64, 64), (128, 128, 128), (64, 128, 256)])
def test_int8_tiles_equal_integer_matmul_with_zero_padding(bm, bn, D):
    rng = np.random.default_rng(bm + bn + D)
    B, H, Hkv, Lq, Lk = 2, 4, 2, 3 * bm - 17, 2 * bn + 5      # ragged both ways
    q, k = _codes(rng, (B, H, Lq, D)), _codes(rng, (B, Hkv, Lk, D))
    tiles = [(0, 0, 0, 0), (1, 3, 2, 2), (1, 2, 1, 0), (0, 1, 2, 1)]
    got = oracle.score_tiles(q, k, bm, bn, "int8", tiles)
    for t, (b, h, qt, kt) in enumerate(tiles):
        kv = h // (H // Hkv)
        a = _pad_block(q[b, h].view(np.int8).astype(np.int64), qt * bm, bm, Lq)
        c = _pad_block(k[b, kv].view(np.int8).astype(np.int64), kt * bn, bn, Lk)
        assert np.array_equal(got[t], (a @ c.T).astype(np.float64)), (b, h, qt, kt)


def test_int8_tile_closed_form_on_ones():
    # every code 1: each entry inside the problem is D, every padded row or key gives 0
    D, bm, bn = 128, 128, 128
    q = np.ones((1, 1, 200, D), np.uint8)
    k = np.ones((1, 1, 150, D), np.uint8)
    t = oracle.score_tiles(q, k, bm, bn, "int8", [(0, 0, 1, 1)])[0]
    assert np.all(t[:72, :22] == D) and np.all(t[72:] == 0) and np.all(t[:, 22:] == 0)
    # -127 * 127 per channel at the extremes of the code range
    q[:] = np.uint8(0x81)  # -127
    k[:] = 127
    t = oracle.score_tiles(q, k, bm, bn, "int8", [(0, 0, 0, 0)])[0]
    assert np.all(t == -127 * 127 * D)


def test_tiles_transpose_symmetry():
    rng = np.random.default_rng(3)
    a, b = _codes(rng, (1, 1, 256, 64)), _codes(rng, (1, 1, 256, 64))
    ab = oracle.score_tiles(a, b, 64, 64, "int8", [(0, 0, 1, 3)])[0]
    ba = oracle.score_tiles(b, a, 64, 64, "int8", [(0, 0, 3, 1)])[0]
    assert np.array_equal(ab, ba.T)


def test_e4m3_tiles_equal_fp64_matmul_of_torch_decoded_codes():
    rng = np.random.default_rng(11)
    D, bm, bn = 128, 128, 128
    q, k = _codes(rng, (1, 2, 140, D)), _codes(rng, (1, 1, 300, D))
    # drop the NaN codes (S.1111.111) so that every code is a number
    q[(q & 0x7F) == 0x7F] = 0x7E
    k[(k & 0x7F) == 0x7F] = 0x7E
    dec = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
    tiles = [(0, 1, 1, 2), (0, 0, 0, 1)]
    got = oracle.score_tiles(q, k, bm, bn, "e4m3", tiles)
    for t, (b, h, qt, kt) in enumerate(tiles):
        a = _pad_block(dec(q[b, h]), qt * bm, bm, 140)
        c = _pad_block(dec(k[b, 0]), kt * bn, bn, 300)
        assert np.array_equal(got[t], a @ c.T)   # every product and partial sum is exact


def test_16bit_tiles_equal_fp64_matmul():
    w = CONFIGS["gqa4k"].replace(B=1, H=4, Hkv=2, Lq=300, Lk=300)
    t = make_workload(w)
    tiles = [(0, 3, 2, 1), (0, 0, 0, 0)]
    got = oracle.score_tiles(t.q, t.k, 128, 128, "16bit", tiles)
    for s, (b, h, qt, kt) in enumerate(tiles):
        a = _pad_block(t.q[b, h].astype(np.float64), qt * 128, 128, 300)
        c = _pad_block(t.k[b, h // 2].astype(np.float64), kt * 128, 128, 300)
        ref = a @ c.T
        assert np.allclose(got[s], ref, rtol=1e-12, atol=1e-9)


def test_bad_tile_list_is_rejected():
    q = np.zeros((1, 2, 64, 64), np.uint8)
    with pytest.raises(ValueError):
        oracle.score_tiles(q, q[:, :1], 64, 64, "int8", [(0, 2, 0, 0)])


# ----------------------------------------------------------------- hint bookkeeping -------

def _adaptive_case():
    w = CONFIGS["adaptive8k"].replace(B=1, H=2, Hkv=1, Lq=640, Lk=640, fmt="int8", tau=2.0)
    t = make_workload(w)
    kw = dict(bm=w.bm, bn=w.bn, causal=True, route="adaptive", fmt="int8", tau=w.tau)
    return w, t, kw


def test_hint_equal_to_own_decisions_changes_nothing():
    w, t, kw = _adaptive_case()
    own = oracle.attention(t.q, t.k, t.v, **kw)
    hinted = oracle.attention(t.q, t.k, t.v, route_hint=own["route"], hint_margin=1e30, **kw)
    assert not hinted["hinted"].any()
    assert np.array_equal(hinted["route"], own["route"])
    assert np.array_equal(hinted["o"], own["o"]) and np.array_equal(hinted["lse"], own["lse"])


def test_flipped_hint_within_margin_is_followed_and_marked():
    # flip the decision of the last live key tile of one query tile (nothing downstream in that
    # query tile depends on it) and set the hint margin just above that decision's margin: the
    # oracle follows the hint there, marks exactly that tile, and nowhere else
    w, t, kw = _adaptive_case()
    own = oracle.attention(t.q, t.k, t.v, **kw)
    r, m = own["route"], own["margin"]
    qt = w.nqt - 1
    kt = int(np.nonzero(r[0, 0, qt])[0].max())
    hint = r.copy()
    hint[0, 0, qt, kt] = 4 - hint[0, 0, qt, kt]          # 1 <-> 3
    hm = float(m[0, 0, qt, kt]) * (1 + 1e-9) + 1e-300
    got = oracle.attention(t.q, t.k, t.v, route_hint=hint, hint_margin=hm, **kw)
    assert got["route"][0, 0, qt, kt] == hint[0, 0, qt, kt]
    marked = np.argwhere(got["hinted"])
    assert marked.tolist() == [[0, 0, qt, kt]]
    # a hint whose margin does not reach the decision is ignored
    got2 = oracle.attention(t.q, t.k, t.v, route_hint=hint, hint_margin=hm * 0.5, **kw)
    assert np.array_equal(got2["route"], r) and not got2["hinted"].any()
