"""Pins of the oracle's routed attention (CPU only).

Each test checks the oracle against something other than itself: hand-solved examples,
brute-force numpy attention (einsum + softmax) on tiny inputs, closed forms (all-8-bit routing
equals exact attention on the dequantised operands, because the per-block scales factor out of
the dot product), invariants (V = 1, causal row 0, permutation of key groups), and
constructed inputs whose adaptive decisions are known by construction.

Sources: TileMix page, section 2 ("Packed Bitmasks", "The Dual-Path Engine": both paths feed
one shared online-softmax state); LampAttention abstract (8-bit products, sensitive
sub-blocks recomputed in 16 bits).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_workload, sample_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- brute force helpers ----

def vis_mask(Lq, Lk, causal, window):
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    if not causal:
        return np.ones((Lq, Lk), bool)
    off = Lk - Lq
    m = j <= i + off
    if window > 0:
        m &= j > i + off - window
    return m


def softmax_attention(s, v, vis):
    """Brute force on a full score matrix s [B,H,Lq,Lk] (fp64), v [B,H,Lk,D]."""
    s = np.where(vis, s, -np.inf)
    M = s.max(-1, keepdims=True)
    empty = ~np.isfinite(M)
    Ms = np.where(empty, 0.0, M)
    p = np.exp(s - Ms)
    l = p.sum(-1, keepdims=True)
    o = np.einsum("bhij,bhjd->bhid", p, v) / np.where(empty, 1.0, l)
    o = np.where(empty, 0.0, o)
    lse = np.where(empty[..., 0], -np.inf, (Ms + np.log(np.where(empty, 1.0, l)))[..., 0])
    return o, lse


def expand_kv(x, H):
    G = H // x.shape[1]
    return np.repeat(x, G, axis=1)


def exact_scores(q, k, scale):
    kk = expand_kv(k.astype(np.float64), q.shape[1])
    return np.einsum("bhid,bhjd->bhij", q.astype(np.float64), kk) * scale


def dequant(codes, scales, blk, fmt):
    if fmt == "int8":
        vals = codes.view(np.int8).astype(np.float64)
    else:
        table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
        vals = table[codes]
    rep = np.repeat(scales.astype(np.float64), blk, axis=-1)[..., : codes.shape[-2]]
    return vals * rep[..., None]


def route_elements(mask, group_tiles, Lq, Lk, bm, bn):
    """Per-element 16-bit selector from the packed mask (bit 0 = 16-bit), [B,H,Lq,Lk]."""
    nkt = -(-Lk // bn)
    kt = np.arange(nkt)
    g = kt // group_tiles
    words = mask[..., g >> 6]  # [B,H,nqt,nkt]
    bits = (words >> (g & 63).astype(np.uint64)) & np.uint64(1)
    sel16 = bits == 0
    sel16 = np.repeat(np.repeat(sel16, bm, axis=2)[:, :, :Lq], bn, axis=3)[..., :Lk]
    return sel16


def rand_qkv(rng, B, H, Hkv, Lq, Lk, D, scale=1.0):
    f = lambda *s: (rng.standard_normal(s) * scale).astype(np.float16).astype(np.float32)
    return f(B, H, Lq, D), f(B, Hkv, Lk, D), f(B, Hkv, Lk, D)


# ------------------------------------------------------------------------- tests ------

def test_hand_examples():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[n], np.float32) for n in ("q", "k", "v"))
        nqt = -(-q.shape[2] // c["bm"])
        nkt = -(-k.shape[2] // c["bn"])
        mask = np.zeros((1, 1, nqt, oracle.mask_words(nkt, 1)), np.uint64)  # all 16-bit
        r = oracle.attention(q, k, v, bm=c["bm"], bn=c["bn"], causal=c["causal"],
                             window=c["window"], scale=c["scale"], mask=mask)
        np.testing.assert_allclose(r["o"], np.array(c["o"]), rtol=0, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(r["lse"], np.array(c["lse"]), rtol=0, atol=1e-14,
                                   err_msg=c["name"])


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 48)])
def test_all_16bit_routing_is_exact_attention(causal, window):
    rng = np.random.default_rng(1)
    B, H, Hkv, Lq, Lk, D, bm, bn = 2, 4, 2, 80, 112, 32, 32, 16
    q, k, v = rand_qkv(rng, B, H, Hkv, Lq, Lk, D)
    nqt, nkt = -(-Lq // bm), -(-Lk // bn)
    mask = np.zeros((B, H, nqt, 1), np.uint64)
    sc = 0.3
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=causal, window=window, scale=sc, mask=mask)
    o, lse = softmax_attention(exact_scores(q, k, sc), expand_kv(v.astype(np.float64), H),
                               vis_mask(Lq, Lk, causal, window))
    np.testing.assert_allclose(r["o"], o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-12)
    live = r["route"] != 0
    assert np.all(r["route"][live] == 2)


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
@pytest.mark.parametrize("causal", [False, True])
def test_all_8bit_routing_is_attention_on_dequantised_operands(fmt, causal):
    rng = np.random.default_rng(2)
    B, H, Hkv, Lq, Lk, D, bm, bn = 1, 2, 1, 96, 96, 64, 32, 32
    q, k, v = rand_qkv(rng, B, H, Hkv, Lq, Lk, D, scale=2.0)
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=causal, scale=0.125, mask=None, fmt=fmt,
                         want_codes=True)
    qd = dequant(r["q_codes"], r["q_scales"], bm, fmt)
    kd = dequant(r["k_codes"], r["k_scales"], bn, fmt)
    o, lse = softmax_attention(exact_scores(qd, kd, 0.125), expand_kv(v.astype(np.float64), H),
                               vis_mask(Lq, Lk, causal, 0))
    np.testing.assert_allclose(r["o"], o, rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-11)
    # and the quantiser inside the attention is the pinned per-block quantiser
    qc, qs = oracle.quantize(q, bm, fmt)
    assert np.array_equal(qc, r["q_codes"]) and np.array_equal(qs, r["q_scales"])


@pytest.mark.parametrize("group_tiles", [1, 2, 3])
def test_mixed_routing_selects_scores_per_tile(group_tiles):
    rng = np.random.default_rng(3)
    B, H, Hkv, Lq, Lk, D, bm, bn = 1, 2, 2, 100, 150, 32, 32, 16
    q, k, v = rand_qkv(rng, B, H, Hkv, Lq, Lk, D, scale=1.5)
    nqt, nkt = -(-Lq // bm), -(-Lk // bn)
    mask = oracle.build_mask(B, H, nqt, nkt, group_tiles, 0.5, 77)
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=True, window=0, scale=0.2, mask=mask,
                         group_tiles=group_tiles, want_codes=True)
    s16 = exact_scores(q, k, 0.2)
    s8 = exact_scores(dequant(r["q_codes"], r["q_scales"], bm, "int8"),
                      dequant(r["k_codes"], r["k_scales"], bn, "int8"), 0.2)
    sel = route_elements(mask, group_tiles, Lq, Lk, bm, bn)
    o, lse = softmax_attention(np.where(sel, s16, s8), expand_kv(v.astype(np.float64), H),
                               vis_mask(Lq, Lk, True, 0))
    np.testing.assert_allclose(r["o"], o, rtol=0, atol=1e-11)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-11)


@pytest.mark.parametrize("route,fmt", [("bitmask", "int8"), ("bitmask", "e4m3"),
                                       ("adaptive", "int8"), ("adaptive", "e4m3")])
def test_v_ones_gives_ones(route, fmt):
    rng = np.random.default_rng(4)
    B, H, Hkv, L, D, bm, bn = 1, 2, 1, 130, 32, 32, 32
    q, k, _ = rand_qkv(rng, B, H, Hkv, L, L, D, scale=3.0)
    v = np.ones_like(k)
    nqt, nkt = -(-L // bm), -(-L // bn)
    mask = oracle.build_mask(B, H, nqt, nkt, 1, 0.4, 1)
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=True, window=40, mask=mask, route=route,
                         fmt=fmt, tau=2.0)
    np.testing.assert_allclose(r["o"], 1.0, rtol=0, atol=1e-13)


@pytest.mark.parametrize("route", ["bitmask", "adaptive"])
def test_causal_row_zero_is_v0(route):
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, 1, 1, 1, 64, 64, 16)
    r = oracle.attention(q, k, v, bm=16, bn=16, causal=True, scale=0.5, route=route, tau=1.0,
                         mask=np.zeros((1, 1, 4, 1), np.uint64), want_codes=True)
    np.testing.assert_allclose(r["o"][0, 0, 0], v[0, 0, 0], rtol=0, atol=1e-15)
    # row 0 sees only key 0: lse = its score, 16-bit in both cases (bitmask all 16-bit;
    # adaptive flags the first live tile)
    s00 = float(np.dot(q[0, 0, 0].astype(np.float64), k[0, 0, 0].astype(np.float64))) * 0.5
    assert abs(r["lse"][0, 0, 0] - s00) < 1e-14


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_key_group_permutation_leaves_output_unchanged(fmt):
    rng = np.random.default_rng(6)
    B, H, Hkv, Lq, D, bm, bn, g = 1, 2, 1, 64, 32, 32, 16, 2
    nkt = 8
    Lk = nkt * bn
    q, k, v = rand_qkv(rng, B, H, Hkv, Lq, Lk, D, scale=2.0)
    nqt = Lq // bm
    mask = oracle.build_mask(B, H, nqt, nkt, g, 0.5, 5)
    perm = np.array([2, 0, 3, 1])  # permutation of the 4 key groups (2 tiles each)
    tile_perm = np.concatenate([[p * g, p * g + 1] for p in perm])
    row_perm = np.concatenate([np.arange(t * bn, (t + 1) * bn) for t in tile_perm])
    k2, v2 = k[:, :, row_perm], v[:, :, row_perm]
    bits = (mask[..., 0][..., None] >> np.arange(4, dtype=np.uint64)) & np.uint64(1)
    bits2 = bits[..., perm]
    mask2 = (bits2 << np.arange(4, dtype=np.uint64)).sum(-1, dtype=np.uint64)[..., None]
    r1 = oracle.attention(q, k, v, bm=bm, bn=bn, mask=mask, group_tiles=g, fmt=fmt)
    r2 = oracle.attention(q, k2, v2, bm=bm, bn=bn, mask=mask2, group_tiles=g, fmt=fmt)
    np.testing.assert_allclose(r1["o"], r2["o"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(r1["lse"], r2["lse"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_adaptive_infinite_tau_is_exact_attention(fmt):
    rng = np.random.default_rng(7)
    B, H, Hkv, L, D, bm, bn = 1, 2, 2, 96, 32, 32, 32
    q, k, v = rand_qkv(rng, B, H, Hkv, L, L, D)
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=True, route="adaptive", fmt=fmt, tau=1e300)
    o, lse = softmax_attention(exact_scores(q, k, 1 / np.sqrt(D)),
                               expand_kv(v.astype(np.float64), H), vis_mask(L, L, True, 0))
    np.testing.assert_allclose(r["o"], o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=0, atol=1e-12)
    live = r["route"] != 0
    assert np.all(r["route"][live] == 3)


@pytest.mark.parametrize("window", [0, 40])
def test_adaptive_very_negative_tau_flags_only_first_visible_tiles(window):
    rng = np.random.default_rng(8)
    L, D, bm, bn = 160, 16, 32, 16
    q, k, v = rand_qkv(rng, 1, 1, 1, L, L, D)
    r = oracle.attention(q, k, v, bm=bm, bn=bn, causal=True, window=window, route="adaptive",
                         tau=-1e300)
    vis = vis_mask(L, L, True, window)
    first = vis.argmax(1)  # first visible key of every row
    nqt, nkt = L // bm, L // bn
    for qt in range(nqt):
        rows = range(qt * bm, (qt + 1) * bm)
        want_flag = {first[i] // bn for i in rows}
        for kt in range(nkt):
            live = vis[qt * bm:(qt + 1) * bm, kt * bn:(kt + 1) * bn].any()
            got = r["route"][0, 0, qt, kt]
            if not live:
                assert got == 0
            else:
                assert got == (3 if kt in want_flag else 1), (qt, kt)


def test_adaptive_constructed_decisions():
    # One query tile of 16 identical rows q = 4*e0; four key tiles whose scores are
    # constant per tile: 0, 5, -10, 4.5 (scale 1).  Known decisions for tau = 1 and 0.4.
    D, bm, bn = 16, 16, 16
    q = np.zeros((1, 1, 16, D), np.float32)
    q[..., 0] = 4.0
    k = np.zeros((1, 1, 64, D), np.float32)
    for t, sc in enumerate([0.0, 5.0, -10.0, 4.5]):
        k[0, 0, t * 16:(t + 1) * 16, 0] = sc / 4.0
        k[0, 0, t * 16:(t + 1) * 16, 1] = 0.25  # keep every key block non-zero
    v = np.random.default_rng(0).standard_normal((1, 1, 64, D)).astype(np.float32)
    for fmt in ("int8", "e4m3"):
        r1 = oracle.attention(q, k, v, bm=bm, bn=bn, scale=1.0, route="adaptive", fmt=fmt, tau=1.0)
        assert r1["route"][0, 0, 0].tolist() == [3, 3, 1, 3]
        r2 = oracle.attention(q, k, v, bm=bm, bn=bn, scale=1.0, route="adaptive", fmt=fmt, tau=0.4)
        assert r2["route"][0, 0, 0].tolist() == [3, 3, 1, 1]
        # margins: tile 2 misses by 5 - 1 - (-10) = 14; tile 3 passes by 4.5 - 4 = 0.5
        assert abs(r1["margin"][0, 0, 0, 2] - 14.0) < 0.2
        assert abs(r1["margin"][0, 0, 0, 3] - 0.5) < 0.2


def test_route_hint_is_followed_only_near_the_threshold():
    D, bm, bn = 16, 16, 16
    q = np.zeros((1, 1, 16, D), np.float32)
    q[..., 0] = 4.0
    k = np.zeros((1, 1, 64, D), np.float32)
    for t, sc in enumerate([0.0, 5.0, -10.0, 4.5]):
        k[0, 0, t * 16:(t + 1) * 16, 0] = sc / 4.0
        k[0, 0, t * 16:(t + 1) * 16, 1] = 0.25
    v = np.ones((1, 1, 64, D), np.float32)
    hint = np.array([[[[1, 1, 3, 1]]]], np.uint8)  # disagrees on tiles 0, 1, 2, 3
    r = oracle.attention(q, k, v, bm=bm, bn=bn, scale=1.0, route="adaptive", tau=1.0,
                         route_hint=hint, hint_margin=0.6)
    # only tile 3 (margin 0.5) is close enough to follow the hint
    assert r["route"][0, 0, 0].tolist() == [3, 3, 1, 1]


@pytest.mark.parametrize("route", ["bitmask", "adaptive"])
def test_sampled_rows_equal_full_rows(route):
    w = CONFIGS["tiny"].replace(Lq=200, Lk=200, H=2, Hkv=1, causal=True, window=0,
                                values="structured", plant_frac=0.02)
    t = make_workload(w)
    mask = oracle.build_mask(w.B, w.H, w.nqt, w.nkt, 1, 0.3, 9)
    kw = dict(bm=w.bm, bn=w.bn, causal=True, mask=mask, route=route, tau=3.0)
    full = oracle.attention(t.q, t.k, t.v, **kw)
    rows = sample_rows(w, 17)
    part = oracle.attention(t.q, t.k, t.v, rows=rows, **kw)
    for b in range(w.B):
        for h in range(w.H):
            np.testing.assert_array_equal(part["o"][b, h], full["o"][b, h, rows[b, h]])
            np.testing.assert_array_equal(part["lse"][b, h], full["lse"][b, h, rows[b, h]])


def test_rows_without_keys_give_zero_and_minus_infinity():
    rng = np.random.default_rng(10)
    q, k, v = rand_qkv(rng, 1, 1, 1, 50, 20, 16)  # bottom-right causal: rows < 30 see nothing
    r = oracle.attention(q, k, v, bm=16, bn=16, causal=True, mask=None)
    assert np.all(r["o"][0, 0, :30] == 0.0)
    assert np.all(np.isneginf(r["lse"][0, 0, :30]))
    assert np.all(np.isfinite(r["lse"][0, 0, 30:]))


def test_error_vs_exact_grows_as_fp16_fraction_falls():
    # TileMix page, section 3 "Numerical Behavior": deviation from the 16-bit reference
    # rises with INT8 coverage.
    w = CONFIGS["tiny"]
    t = make_workload(w)
    ex = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn,
                          mask=np.zeros((1, 1, w.nqt, 1), np.uint64))
    errs = []
    for p in (1.0, 0.75, 0.5, 0.25, 0.0):
        m = oracle.build_mask(1, 1, w.nqt, w.nkt, 1, p, 3)
        r = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, mask=m)
        errs.append(np.abs(r["o"] - ex["o"]).mean())
    assert errs[0] == 0.0
    assert all(a < b for a, b in zip(errs, errs[1:]))


def test_tiny_golden_record_is_reproduced():
    """Regression record of the oracle on the tiny workload (tests/golden/make_golden.py)."""
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        g = json.load(f)
    w = CONFIGS["tiny"]
    t = make_workload(w)
    mask = oracle.build_mask(w.B, w.H, w.nqt, w.nkt, w.group_tiles, w.p_fp16, w.mask_seed)
    assert [str(int(x)) for x in mask.reshape(-1)] == g["mask"]
    r = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, mask=mask, group_tiles=w.group_tiles,
                         fmt=w.fmt, want_codes=True)
    assert r["route"].reshape(-1).tolist() == g["route"]
    assert [float(x) for x in r["q_scales"].reshape(-1)] == g["q_scales"]
    assert [float(x) for x in r["k_scales"].reshape(-1)] == g["k_scales"]
    assert int(r["q_codes"].view(np.int8).astype(np.int64).sum()) == g["q_code_sum"]
    np.testing.assert_allclose(r["lse"].reshape(-1), g["lse"], rtol=0, atol=1e-12)
    for idx, val in g["o_samples"]:
        assert abs(r["o"][tuple(idx)] - val) < 1e-12
    assert abs(np.abs(r["o"]).sum() - g["o_abs_sum"]) < 1e-9


# ---- threshold skip (LATTE page: low-precision filtering of keys far below the row max) ----

def _skip_case():
    # One query tile of 16 identical rows q = 4*e0; four key tiles with constant scores per tile
    # 6, 0, -30, 1 (scale 1): the running max after tile 0 is 6.
    D, bm, bn = 16, 16, 16
    q = np.zeros((1, 1, 16, D), np.float32)
    q[..., 0] = 4.0
    k = np.zeros((1, 1, 64, D), np.float32)
    for t, sc in enumerate([6.0, 0.0, -30.0, 1.0]):
        k[0, 0, t * 16:(t + 1) * 16, 0] = sc / 4.0
        k[0, 0, t * 16:(t + 1) * 16, 1] = 0.25
    v = np.random.default_rng(1).standard_normal((1, 1, 64, D)).astype(np.float32)
    return q, k, v, bm, bn


def test_skip_drops_exactly_the_tiles_below_the_threshold():
    q, k, v, bm, bn = _skip_case()
    for fmt in ("int8", "e4m3"):
        # tau huge: every kept tile is recomputed in 16 bits, so the output is plain attention
        # over the kept keys; skip_tau 20 drops tile 2 only (-30 < 6 - 20; 0 and 1 are not)
        r = oracle.attention(q, k, v, bm=bm, bn=bn, scale=1.0, route="adaptive", fmt=fmt,
                             tau=1e9, skip_tau=20.0)
        assert r["route"][0, 0, 0].tolist() == [3, 3, 4, 3]
        keep = np.ones(64, bool)
        keep[32:48] = False
        s = exact_scores(q, k, 1.0)[..., keep]
        o, lse = softmax_attention(s, v[:, :, keep].astype(np.float64), np.ones((16, 48), bool))
        assert np.abs(r["o"] - o).max() < 1e-12 and np.abs(r["lse"] - lse).max() < 1e-12
        # skip_tau 5.5 also drops tile 1 (0 < 6 - 5.5) but keeps tile 3 (1 >= 0.5)
        r = oracle.attention(q, k, v, bm=bm, bn=bn, scale=1.0, route="adaptive", fmt=fmt,
                             tau=1e9, skip_tau=5.5)
        assert r["route"][0, 0, 0].tolist() == [3, 4, 4, 3]
        # margins: tile 2 dropped by 6 - 5.5 + 30 = 30.5; tile 3 kept by 1 - 0.5 = 0.5
        assert abs(r["margin"][0, 0, 0, 2] - 30.5) < 0.3
        assert abs(r["margin"][0, 0, 0, 3] - 0.5) < 0.3


def test_skip_infinite_threshold_changes_nothing_and_first_tiles_stay():
    rng = np.random.default_rng(5)
    q, k, v = rand_qkv(rng, 1, 2, 1, 200, 200, 64, scale=1.5)
    kw = dict(bm=64, bn=64, causal=True, route="adaptive", fmt="int8", tau=2.0)
    a = oracle.attention(q, k, v, **kw)
    b = oracle.attention(q, k, v, skip_tau=float("inf"), **kw)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["route"], b["route"])
    # even skip_tau = 0 never drops a query tile's first live key tile (no running max yet),
    # so every row keeps some key and its lse stays finite
    c = oracle.attention(q, k, v, skip_tau=0.0, **kw)
    assert (c["route"] == 4).any()
    for qt in range(c["route"].shape[2]):
        live = np.nonzero(c["route"][0, 0, qt])[0]
        assert c["route"][0, 0, qt, live[0]] != 4
    assert np.isfinite(c["lse"]).all()


# ---- 8-bit key cache (TileMix page, section 4: INT8 key/value caches for decode) ----------

def test_key_cache_codes_are_used_as_given():
    # one query row q = 2 * e0 (codes [127, 0, ...], scale fl32(2/127)); a hand-made cache of 4
    # keys with codes 10, -20, 30, 0 on channel 0 and block scale 0.5: the 8-bit scores are
    # 127 * c_j * fl32(2/127) * 0.5 (scale 1); v is given as dequantised values
    D = 16
    q = np.zeros((1, 1, 1, D), np.float32)
    q[0, 0, 0, 0] = 2.0
    codes = np.zeros((1, 1, 4, D), np.uint8)
    codes[0, 0, :, 0] = np.array([10, -20, 30, 0], np.int8).view(np.uint8)
    ks = np.array([[[0.5]]], np.float32)
    k_values = codes.view(np.int8).astype(np.float32) * 0.5  # the cache, dequantised
    v = np.random.default_rng(3).standard_normal((1, 1, 4, D)).astype(np.float32)
    r = oracle.attention(q, k_values, v, bm=1, bn=4, scale=1.0, k_codes_in=codes, k_scales_in=ks)
    sq = float(np.float32(2.0) / np.float32(127.0))
    s = 127.0 * np.array([10.0, -20.0, 30.0, 0.0]) * sq * 0.5
    p = np.exp(s - s.max())
    assert np.allclose(r["o"][0, 0, 0], (p[:, None] * v[0, 0]).sum(0) / p.sum(), atol=1e-12)
    assert abs(r["lse"][0, 0, 0] - (s.max() + np.log(p.sum()))) < 1e-12


def test_key_cache_equal_to_own_quantisation_changes_nothing():
    rng = np.random.default_rng(9)
    q, k, v = rand_qkv(rng, 1, 4, 2, 1, 300, 64, scale=1.5)
    kc, ksc = oracle.quantize(k, 64, "int8")
    m = oracle.build_mask(1, 4, 1, 5, 1, 0.3, 11)
    kw = dict(bm=64, bn=64, causal=True, mask=m, group_tiles=1)
    a = oracle.attention(q, k, v, **kw)
    b = oracle.attention(q, k, v, k_codes_in=kc, k_scales_in=ksc, **kw)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["lse"], b["lse"])
