"""Host-side routing-template arithmetic of the library (no GPU): the 16-bit pair fraction
of a structured template and the search for a target INT8 share (TileMix page, section 3:
the 75%-INT8 "SpTrans75" configuration; section 4: static, data-free structured templates),
checked against brute force on the oracle's template bits."""
import itertools

import numpy as np
import pytest

import mixed_precision_tiled_b200 as mpt
import oracle


def brute_fraction(Lq, Lk, D, gt, causal, window, sink, band, stride):
    bm, bn = mpt.lamp_tile_shape(D)
    m = oracle.build_mask_template(1, 1, Lq, Lk, bm, bn, gt, sink, band, stride)[0, 0]
    tot = six = 0
    for i in range(Lq):
        for j in range(Lk):
            if causal and (j > i + Lk - Lq or (window > 0 and j <= i + Lk - Lq - window)):
                continue
            g = (j // bn) // gt
            bit = (int(m[i // bm][g >> 6]) >> (g & 63)) & 1
            tot += 1
            six += bit == 0
    return six / tot if tot else 0.0


@pytest.mark.parametrize("Lq,Lk,D,gt,causal,window", [
    (512, 512, 64, 1, 1, 0), (300, 700, 128, 2, 1, 0), (700, 300, 64, 3, 1, 0),
    (640, 640, 256, 2, 1, 200), (384, 512, 128, 1, 0, 0)])
def test_template_fraction_matches_brute_force(Lq, Lk, D, gt, causal, window):
    for sink, band, stride in [(0, 1, 0), (1, 2, 3), (2, 1, 2), (0, 0, 0), (1, 3, 0)]:
        got = mpt.lamp_template_fraction(Lq, Lk, D, gt, causal, window, sink, band, stride)
        want = brute_fraction(Lq, Lk, D, gt, causal, window, sink, band, stride)
        assert got == pytest.approx(want, abs=1e-12), (sink, band, stride)


def test_template_search_is_the_first_best_of_its_grid():
    Lq = Lk = 2048
    D, gt, causal, window, target = 64, 2, 1, 0, 0.75
    sink, band, stride, fr = mpt.lamp_template_for_int8_fraction(Lq, Lk, D, gt, causal, window,
                                                                  target)
    assert fr == pytest.approx(mpt.lamp_template_fraction(Lq, Lk, D, gt, causal, window, sink,
                                                          band, stride), abs=1e-12)
    ng = -(-(Lk // 64) // gt)
    best = None
    for s in (1, 0):
        for st in [0] + list(range(2, ng + 1)):
            for b in range(1, ng + 1):
                f = mpt.lamp_template_fraction(Lq, Lk, D, gt, causal, window, s, b, st)
                if best is None or abs(f - (1 - target)) < best[0] - 1e-12:
                    best = (abs(f - (1 - target)), s, b, st)
    assert (sink, band, stride) == best[1:]


def test_sptrans75_at_the_workload_shapes():
    # a 75% INT8 template exists within half a percent at the long-context shapes
    for L, gt in [(4096, 4), (32768, 8), (131072, 8)]:
        _, _, _, fr = mpt.lamp_template_for_int8_fraction(L, L, 128, gt, 1, 0, 0.75)
        assert abs(fr - 0.25) < 0.005, (L, fr)
