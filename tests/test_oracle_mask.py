"""Pins of the oracle's routing-mask templates (CPU only): the seeded Bernoulli template and
the structured static template.

Mask layout and polarity follow the TileMix page, section 2 "Packed Bitmasks": one bit per
group of adjacent key tiles, 0 = FP16, 1 = INT8.  The bits are drawn from SplitMix64, pinned
here to the generator's published reference outputs.
"""
import json
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


# ---- structured static routing template (TileMix page, sections 3 and 4) ----------------

def _template_bits(m, ng):
    return ["".join(str((int(w[g >> 6]) >> (g & 63)) & 1) for g in range(ng)) for w in m]


def test_template_matches_hand_derived_tables():
    with open(os.path.join(GOLDEN, "mask_template_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        m = oracle.build_mask_template(c["B"], c["H"], c["Lq"], c["Lk"], c["bm"], c["bn"],
                                       c["group_tiles"], c["sink"], c["band"], c["stride"])
        ng = len(c["bits"][0])
        assert _template_bits(m[0, 0], ng) == c["bits"], c["name"]


def test_template_extremes():
    # band covering every group -> all FP16; nothing selected -> every group INT8;
    # stride 1 divides every distance -> all FP16; unused bits stay 0
    L, bm, gt = 4096, 128, 1
    ng = L // bm
    full = oracle.build_mask_template(1, 2, L, L, bm, bm, gt, 0, ng, 0)
    assert not full.any()
    none = oracle.build_mask_template(1, 2, L, L, bm, bm, gt, 0, 0, 0)
    assert np.all(none == np.uint64((1 << ng) - 1))
    s1 = oracle.build_mask_template(1, 2, L, L, bm, bm, gt, 0, 0, 1)
    assert not s1.any()
    # 130 groups need three words; bits 130..191 are zero
    big = oracle.build_mask_template(1, 1, 130 * 128, 130 * 128, 128, 128, 1, 0, 0, 0)
    assert big.shape[-1] == 3 and int(big[0, 0, 0, 2]) == 0b11


def test_template_is_a_band_around_the_diagonal():
    # with sink 0 and no stride, row qt's FP16 groups are exactly those within band - 1 of gd;
    # every (b, h) gets the same data-free template
    L, bm, gt, band = 8192, 128, 4, 3
    m = oracle.build_mask_template(2, 3, L, L, bm, bm, gt, 0, band, 0)
    ng = L // bm // gt
    for qt in range(L // bm):
        gd = qt // gt
        want = "".join("0" if abs(gd - g) < band else "1" for g in range(ng))
        assert _template_bits(m[1, 2, qt:qt + 1], ng)[0] == want
    assert np.array_equal(m[0, 0], m[1, 2])
