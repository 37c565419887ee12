"""Pins of the oracle's 8-bit exponentials and 8-bit P.V (CPU).

Reading (LampAttention abstract: exponentials in 8-bit formats; the pages fix no format): V in
E4M3 with one scale per (batch, KV head, channel) over all keys; every p = e^(s - m_t) * 2^8
rounded to E4M3 against the running max m_t after its key tile (ascending tiles); O = sv *
sum p8 v8 / sum p8 over the tiles rescaled to the final max; lse stays the exact softmax's.
Pinned here against torch's e4m3 conversion, the pinned e4m3 encoder, closed forms (constant
V, a single visible key) and a hand-worked example whose second key tile raises the max.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _e4m3_values():
    return np.array([oracle.e4m3_decode(c) for c in range(0x00, 0x7F)], dtype=np.float64)


def test_round_pos_equals_the_pinned_encoder():
    rng = np.random.default_rng(5)
    vals = _e4m3_values()
    mids = (vals[:-1] + vals[1:]) / 2
    xs = np.concatenate([vals, mids, rng.uniform(0, 256, 4000), 2.0 ** rng.uniform(-12, 8, 4000)])
    xs = xs.astype(np.float32).astype(np.float64)  # values the fp32 encoder sees exactly
    for x in xs:
        r, d = oracle.e4m3_round_pos(x)
        assert r == oracle.e4m3_decode(oracle.e4m3_encode(x)), x
        assert d >= 0.0
    for m in mids:
        assert oracle.e4m3_round_pos(m)[1] == 0.0  # exactly on a midpoint
    # on a grid point the distance is half a step over the value
    assert oracle.e4m3_round_pos(96.0)[1] == pytest.approx(0.5 * 8 / 96)
    assert oracle.e4m3_round_pos(2.0 ** -8)[1] == pytest.approx(0.5 * 2 ** -9 / 2 ** -8)
    assert oracle.e4m3_round_pos(0.0) == (0.0, math.inf)


def test_quantize_v_per_channel():
    rng = np.random.default_rng(9)
    v = rng.standard_normal((2, 3, 50, 8)).astype(np.float32)
    v[1, 2, :, 5] = 0.0                                  # an all-zero channel
    codes, scales = oracle.quantize_v(v)
    assert codes.shape == (2, 3, 8, 50) and scales.shape == (2, 3, 8)
    a = np.abs(v).max(axis=2)                            # [2, 3, 8]
    expect_s = np.where(a == 0, 0, (a / np.float32(448)).astype(np.float32))
    assert np.array_equal(scales, expect_s)
    assert scales[1, 2, 5] == 0 and np.all(codes[1, 2, 5] == 0)
    # codes = torch's round-to-nearest-even e4m3 of fl32(v / s), channel-major
    s = np.where(scales == 0, 1, scales)[:, :, None, :]
    y = (v / s).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref = np.where((scales == 0)[:, :, None, :], 0, ref)
    assert np.array_equal(codes, np.swapaxes(ref, 2, 3))
    # the channel's absmax element gets the largest code
    j = np.abs(v[0, 0, :, 3]).argmax()
    assert codes[0, 0, 3, j] & 0x7F == 0x7E
    # a power-of-two scaling of V leaves the codes and scales the scales
    c2, s2 = oracle.quantize_v(v * np.float32(8))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales * 8)


def _run(q, k, v, **kw):
    return oracle.attention(q, k, v, pv8=True, **kw)


def test_constant_v_gives_its_quantised_value():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 2, 40, 16)).astype(np.float32)
    k = rng.standard_normal((1, 1, 40, 16)).astype(np.float32)
    u = rng.standard_normal(16).astype(np.float32)
    v = np.broadcast_to(u, (1, 1, 40, 16)).copy()
    out = _run(q, k, v, bm=8, bn=8, causal=True)
    s = out["v_scales"][0, 0]
    expect = np.sign(u).astype(np.float64) * 448.0 * s.astype(np.float64)
    # the p8 weights cancel; only the fp64 rescales of a rising max leave rounding behind
    assert np.allclose(out["o"][0, 0], np.broadcast_to(expect, (40, 16)), rtol=1e-14, atol=0)


def test_single_visible_key_gives_its_value():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 20, 8)).astype(np.float32)
    k = rng.standard_normal((1, 1, 20, 8)).astype(np.float32)
    v = rng.standard_normal((1, 1, 20, 8)).astype(np.float32)
    out = _run(q, k, v, bm=4, bn=4, causal=True)
    exact = oracle.attention(q, k, v, bm=4, bn=4, causal=True)
    codes, scales = out["v_codes"][0, 0], out["v_scales"][0, 0]
    v8 = np.array([oracle.e4m3_decode(c) for c in codes[:, 0]]) * scales.astype(np.float64)
    assert np.array_equal(out["o"][0, 0, 0], v8)        # row 0 sees key 0 only
    assert np.array_equal(out["lse"], exact["lse"])     # lse is the exact softmax's


def test_hand_worked_two_tiles_with_a_rising_max():
    # one query, four keys in key tiles of two; 16-bit routing (mask bits 0) so the scores are
    # the exact products: s = [0, -1, 1.5, -6.5].  Tile 0 against m_0 = 0: p = 256 and 256 e^-1
    # = 94.18 -> 96 (E4M3 step 8 on [64, 128)); tile 1 against m_1 = 1.5: p = 256 and 256 e^-8 =
    # 0.08588 -> 0.0859375 (step 2^-7 on [2^-4, 2^-3); without the 2^8 it would fall below the
    # subnormal grid and round to 0).  V channel 0 = [448, 224, 112, 56] (exact E4M3 values,
    # scale fl32(448 / 448) = 1); channels 1-3 are zero.
    q = np.zeros((1, 1, 1, 4), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 4, 4), np.float32)
    k[0, 0, :, 0] = [0.0, -1.0, 1.5, -6.5]
    v = np.zeros((1, 1, 4, 4), np.float32)
    v[0, 0, :, 0] = [448.0, 224.0, 112.0, 56.0]
    mask = np.zeros((1, 1, 1, 1), np.uint64)              # every group 16-bit
    out = _run(q, k, v, bm=1, bn=2, scale=1.0, mask=mask)
    f = math.exp(0.0 - 1.5)                               # tile 0 rescaled to the final max
    num = f * (256 * 448 + 96 * 224) + 256 * 112 + 0.0859375 * 56
    den = f * (256 + 96) + 256 + 0.0859375
    assert out["o"][0, 0, 0, 0] == pytest.approx(num / den, rel=1e-15)
    assert np.all(out["o"][0, 0, 0, 1:] == 0)
    # the row's smallest distance from a rounding midpoint, over its four p
    def dist(p, step):
        return abs(p / step - math.floor(p / step) - 0.5) * step / p
    expect = min(dist(256.0, 32), dist(256 * math.exp(-1.0), 8), dist(256 * math.exp(-8.0), 2 ** -7))
    assert out["pv8_margin"][0, 0, 0] == pytest.approx(expect)


def test_close_to_exact_attention_within_the_rounding_bound():
    # every p is within half an E4M3 step (2^-4 relative on the normal range, 2^-10 absolute
    # below 2^-6) of its exact value, and V within half a step of its per-channel grid
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 2, 96, 32)).astype(np.float32)
    k = rng.standard_normal((1, 1, 96, 32)).astype(np.float32)
    v = rng.standard_normal((1, 1, 96, 32)).astype(np.float32)
    mask = np.zeros((1, 2, 3, 1), np.uint64)              # 16-bit scores: isolate P and V
    pv = _run(q, k, v, bm=32, bn=32, causal=True, mask=mask)
    ex = oracle.attention(q, k, v, bm=32, bn=32, causal=True, mask=mask)
    vmax = np.abs(v).max()
    err = np.abs(pv["o"] - ex["o"]).max()
    assert err < 2 * (2.0 ** -4) * vmax and err > 0
    assert np.array_equal(pv["lse"], ex["lse"])
