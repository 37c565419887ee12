"""Pins of the oracle's per-block quantiser and e4m3 codec (CPU only).

The quantiser follows the TileMix page, section 2 "The Dual-Path Engine" (INT8 path with
per-block scale factors) and the LampAttention abstract (8-bit formats); the block size,
absmax/127 scale and round-half-even come from the workload definition.  None of these tests
restates the oracle's code: they check properties that any correct per-block absmax
quantiser must have, and the e4m3 codec against torch's float8_e4m3fn.
"""
import numpy as np
import pytest
import torch

import oracle


def _blocks(x, blk):
    L = x.shape[-2]
    for b0 in range(0, L, blk):
        yield b0, min(L, b0 + blk)


def _int8(codes):
    return codes.view(np.int8).astype(np.int64)


@pytest.mark.parametrize("L,blk,D", [(256, 64, 64), (200, 64, 32), (130, 128, 16), (1, 64, 8)])
def test_int8_round_to_nearest_and_absmax(L, blk, D):
    rng = np.random.default_rng(L * 7 + D)
    x = (rng.standard_normal((2, L, D)) * rng.uniform(0.01, 50, size=(2, L, 1))).astype(np.float32)
    codes, s = oracle.quantize(x, blk, "int8")
    c = _int8(codes)
    assert s.shape == (2, -(-L // blk))
    for o in range(2):
        for bi, (r0, r1) in enumerate(_blocks(x, blk)):
            blkx = x[o, r0:r1].astype(np.float64)
            sc = float(s[o, bi])
            a = np.abs(blkx).max()
            # scale is absmax / 127 rounded to fp32
            assert abs(sc - a / 127.0) <= a / 127.0 * 2 ** -23
            cb = c[o, r0:r1]
            assert cb.min() >= -127 and cb.max() <= 127
            # the absmax element maps to +-127
            i = np.unravel_index(np.abs(blkx).argmax(), blkx.shape)
            assert abs(cb[i]) == 127 and np.sign(cb[i]) == np.sign(blkx[i])
            # nearest code: |x - c*s| <= s/2 (up to the fp32 rounding of x/s)
            err = np.abs(blkx - cb * sc)
            assert np.all(err <= sc * (0.5 + 2 ** -20))


def test_int8_ties_go_to_even_and_division_is_exact():
    # absmax 127 makes the scale exactly 1, so x/s = x and the ties are exact halves
    x = np.zeros((1, 4, 8), np.float32)
    x[0, 0, :] = [127, 0.5, 1.5, 2.5, -2.5, -3.5, 126.5, -0.5]
    x[0, 1, :] = [4.5, 5.5, -4.5, 0.49999997, 1.0000001, 63.5, 64.5, -126.5]
    codes, s = oracle.quantize(x, 4, "int8")
    assert s[0, 0] == np.float32(1.0)
    c = _int8(codes)[0]
    assert c[0].tolist() == [127, 0, 2, 2, -2, -4, 126, 0]
    assert c[1].tolist() == [4, 6, -4, 0, 1, 64, 64, -126]


def test_int8_power_of_two_scaling_leaves_codes_unchanged():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 96, 32)).astype(np.float32)
    c0, s0 = oracle.quantize(x, 32, "int8")
    for k in (-7, -1, 3, 10):
        c1, s1 = oracle.quantize(x * np.float32(2.0 ** k), 32, "int8")
        assert np.array_equal(c0, c1)
        assert np.array_equal(s1, s0 * np.float32(2.0 ** k))


def test_zero_block_and_block_isolation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 192, 16)).astype(np.float32)
    x[0, 64:128] = 0.0
    for fmt in ("int8", "e4m3"):
        c, s = oracle.quantize(x, 64, fmt)
        assert s[0, 1] == 0.0 and not c[0, 64:128].any()
        # changing one block leaves the others' codes and scales alone
        y = x.copy()
        y[0, 130, 3] = 1000.0
        c2, s2 = oracle.quantize(y, 64, fmt)
        assert np.array_equal(c[0, :128], c2[0, :128]) and np.array_equal(s[0, :2], s2[0, :2])
        assert s2[0, 2] != s[0, 2]


def test_ragged_last_block_uses_only_its_rows():
    x = np.ones((1, 70, 4), np.float32)
    x[0, :64] *= 100.0
    c, s = oracle.quantize(x, 64, "int8")
    assert s.shape == (1, 2)
    assert s[0, 1] == np.float32(1.0) / np.float32(127.0)
    assert np.all(_int8(c)[0, 64:] == 127)


# ---------------------------------------------------------------- e4m3 codec ----------

def _torch_decode_all():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_for_all_codes():
    ref = _torch_decode_all()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encode_round_trips_every_code_and_ties_to_even():
    ref = _torch_decode_all()
    finite = [c for c in range(256) if not np.isnan(ref[c])]
    for c in finite:
        e = oracle.e4m3_encode(np.float32(ref[c]))
        # +0 and -0 both decode to 0; the encoder keeps the sign bit
        assert e == c, (c, e)
    # midpoints between neighbouring positive codes go to the even mantissa
    pos = [c for c in range(0x00, 0x7F)]
    for c in pos[:-1]:
        lo, hi = ref[c], ref[c + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # exact in fp32
        want = c if (c & 1) == 0 else c + 1
        assert oracle.e4m3_encode(mid) == want
        assert oracle.e4m3_encode(-mid) == want | 0x80


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000) * 60, rng.uniform(-448, 448, 20000),
                        rng.standard_normal(5000) * 1e-3]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], dtype=np.uint8)
    assert np.array_equal(ref, got)
    for big in (448.0, 449.0, 463.9, 464.0, 1e4, 3.0e38):
        assert oracle.e4m3_encode(big) == 0x7E
        assert oracle.e4m3_encode(-big) == 0xFE


def test_e4m3_quantiser_scale_and_nearest():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((2, 128, 64)) * 3).astype(np.float32)
    codes, s = oracle.quantize(x, 64, "e4m3")
    dec = _torch_decode_all()
    for o in range(2):
        for bi, (r0, r1) in enumerate(_blocks(x, 64)):
            blkx = x[o, r0:r1].astype(np.float64)
            a = np.abs(blkx).max()
            sc = float(s[o, bi])
            assert abs(sc - a / 448.0) <= a / 448.0 * 2 ** -23
            vals = dec[codes[o, r0:r1]]
            # absmax maps to +-448
            i = np.unravel_index(np.abs(blkx).argmax(), blkx.shape)
            assert abs(vals[i]) == 448.0
            # nearest e4m3 value of x/s: no other code is closer
            y = (blkx / sc)
            fin = dec[~np.isnan(dec)]
            best = np.abs(y[..., None] - fin[None, None, :]).min(-1)
            assert np.all(np.abs(y - vals) <= best + 1e-6 * np.abs(y) + 1e-12)
