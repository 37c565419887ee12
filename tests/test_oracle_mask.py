"""Pins of the oracle's routing-mask template (CPU only).

Mask layout and polarity follow the TileMix page, section 2 "Packed Bitmasks": one bit per
group of adjacent key tiles, 0 = FP16, 1 = INT8.  The bits are drawn from SplitMix64, pinned
here to the generator's published reference outputs.
"""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


def test_splitmix64_reference_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        want = [int(l) for l in f if l.strip() and not l.startswith("#")]
    state, got = 1234567, []
    for _ in range(len(want)):
        got.append(oracle.splitmix64_next(state))
        state = (state + GAMMA) & M64
    assert got == want


def test_mask_extremes_and_unused_bits():
    # p_fp16 = 0: every live group 8-bit ("One"); p_fp16 = 1: all FP16 (exact attention)
    m0 = oracle.build_mask(2, 3, 5, 70, 1, 0.0, 42)
    assert m0.shape == (2, 3, 5, 2)
    assert np.all(m0[..., 0] == np.uint64(M64))
    assert np.all(m0[..., 1] == np.uint64((1 << 6) - 1))  # 70 groups: bits >= 70 stay 0
    m1 = oracle.build_mask(2, 3, 5, 70, 1, 1.0, 42)
    assert not m1.any()


def test_mask_fraction_is_bernoulli():
    B, H, nqt, nkt, g, p = 1, 8, 64, 64, 2, 0.3
    m = oracle.build_mask(B, H, nqt, nkt, g, p, 7)
    ng = 32
    bits = (m[..., 0][..., None] >> np.arange(ng, dtype=np.uint64)) & np.uint64(1)
    frac_fp16 = 1.0 - bits.mean()
    n = B * H * nqt * ng
    assert abs(frac_fp16 - p) < 5 * np.sqrt(p * (1 - p) / n)


def test_mask_bits_are_independent_draws_per_group_index():
    # Bit g of (b, h, qt) depends only on the flat group index and the seed: the same index
    # under a different (B, H) split gives the same bit, and a different seed changes it.
    a = oracle.build_mask(1, 4, 8, 16, 1, 0.5, 99)
    b = oracle.build_mask(2, 2, 8, 16, 1, 0.5, 99)
    assert np.array_equal(a.reshape(-1), b.reshape(-1))
    c = oracle.build_mask(1, 4, 8, 16, 1, 0.5, 100)
    assert not np.array_equal(a, c)


def test_mask_draw_matches_threshold_on_generator_output():
    # bit = 0 (FP16) iff the top 53 bits of the hash, as a fraction, fall below p
    B, H, nqt, nkt, g, p, seed = 1, 1, 3, 10, 3, 0.4, 5
    ng = -(-nkt // g)
    m = oracle.build_mask(B, H, nqt, nkt, g, p, seed)
    for qt in range(nqt):
        for gi in range(ng):
            idx = qt * ng + gi
            u = oracle.splitmix64_next(seed ^ ((idx * GAMMA) & M64))
            want = 0 if (u >> 11) * 2.0 ** -53 < p else 1
            assert (int(m[0, 0, qt, 0]) >> gi) & 1 == want
