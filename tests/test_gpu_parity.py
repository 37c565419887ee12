"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on seeded inputs.

Small cases span several tiles and a ragged tail and are compared element by element; the
full-size workloads are compared on seeded samples of query rows (bitmask routing: rows are
independent) or whole query tiles (adaptive routing: a tile's decisions depend on all its
rows), in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
import oracle
from workloads import CONFIGS, make_workload, sample_rows, sample_tiles, to_16bit

from _parity import (EXACT_MAX_ABS, check_outputs, gpu_run, mask_to_numpy, oracle_run,
                     parity_case, to_dev)

pytestmark = pytest.mark.gpu

TINY = CONFIGS["tiny"]
GQA = CONFIGS["gqa4k"]


def small(base, **kw):
    return base.replace(**kw)


# ----------------------------------------------------------------- quantiser / mask ----

@pytest.mark.parametrize("D,L,dtype,fmt", [(64, 256, "fp16", "int8"), (128, 600, "bf16", "int8"),
                                           (128, 600, "bf16", "e4m3"), (256, 200, "bf16", "int8"),
                                           (256, 130, "fp16", "e4m3")])
def test_quantiser_bit_exact(D, L, dtype, fmt):
    bm, bn = mpt.lamp_tile_shape(D)
    w = small(GQA, D=D, Lq=L, Lk=L, B=2, H=4, Hkv=2, bm=bm, bn=bn, dtype=dtype)
    t = make_workload(w)
    q, k = to_dev(t.q_bits, dtype), to_dev(t.k_bits, dtype)
    q8, k8, qs, ks = mpt.quantize(q, k, fmt=fmt)
    torch.cuda.synchronize()
    rq, rqs = oracle.quantize(t.q, bm, fmt)
    rk, rks = oracle.quantize(t.k, bn, fmt)
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(qs.cpu().numpy(), rqs)
    assert np.array_equal(k8.cpu().numpy(), rk) and np.array_equal(ks.cpu().numpy(), rks)


@pytest.mark.parametrize("name", ["gqa4k", "gemma_local16k", "long32k"])
def test_quantiser_bit_exact_full_size(name):
    w = CONFIGS[name]
    t = make_workload(w)
    q, k = to_dev(t.q_bits, w.dtype), to_dev(t.k_bits, w.dtype)
    q8, k8, qs, ks = mpt.quantize(q, k, fmt=w.fmt)
    torch.cuda.synchronize()
    rq, rqs = oracle.quantize(t.q, w.bm, w.fmt)
    rk, rks = oracle.quantize(t.k, w.bn, w.fmt)
    assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(ks.cpu().numpy(), rks)
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(k8.cpu().numpy(), rk)


def test_quantiser_e4m3_full_size_adaptive_workload():
    w = CONFIGS["adaptive8k"]
    t = make_workload(w)
    q, k = to_dev(t.q_bits, w.dtype), to_dev(t.k_bits, w.dtype)
    q8, k8, qs, ks = mpt.quantize(q, k, fmt="e4m3")
    torch.cuda.synchronize()
    rk, rks = oracle.quantize(t.k, w.bn, "e4m3")
    assert np.array_equal(ks.cpu().numpy(), rks) and np.array_equal(k8.cpu().numpy(), rk)
    rq, rqs = oracle.quantize(t.q, w.bm, "e4m3")
    assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(q8.cpu().numpy(), rq)


def _edge_blocks(fmt, dtype, D=128, L=600, seed=5):
    """Blocks of 128 rows that stress the quantiser's rounding: exact ties of the 8-bit format
    (absmax chosen so that the scale is 1), an all-zero block, a block of subnormal values (a
    subnormal scale), a normal random block and a ragged last block."""
    rng = np.random.default_rng(seed)
    top = 127.0 if fmt == "int8" else 448.0
    x = np.zeros((1, 1, L, D), np.float32)
    if fmt == "int8":
        ties = rng.integers(-127, 127, size=(128, D)) + 0.5   # half-integers: round to even
    else:
        grid = np.array([1.0625, 17.0, 1.5 * 2.0 ** -9, 0.3125 * 2 ** -4, 208.0, 3.75])
        ties = rng.choice(grid, size=(128, D)) * rng.choice([-1.0, 1.0], size=(128, D))
    ties[0, 0] = top                                          # absmax -> scale exactly 1
    x[0, 0, 0:128] = ties
    # rows 128..255 stay zero
    x[0, 0, 256:384] = rng.standard_normal((128, D)) * 2.0 ** -130   # subnormal in fp32 / bf16
    x[0, 0, 384:512] = rng.standard_normal((128, D)) * np.exp(rng.standard_normal((128, D)))
    x[0, 0, 512:] = rng.standard_normal((L - 512, D)) * 3.0
    if dtype == "fp16":
        x[0, 0, 256:384] = rng.standard_normal((128, D)) * 2.0 ** -20  # fp16 subnormals
    bits, vals = to_16bit(x, dtype)
    return bits, vals


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_quantiser_rounding_edge_blocks(fmt, dtype):
    bits, vals = _edge_blocks(fmt, dtype)
    q = to_dev(bits, dtype)
    q8, k8, qs, ks = mpt.quantize(q, q, fmt=fmt)
    torch.cuda.synchronize()
    rq, rqs = oracle.quantize(vals, 128, fmt)
    assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(ks.cpu().numpy(), rqs)
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(k8.cpu().numpy(), rq)
    assert rqs[0, 0, 1] == 0 and 0 < rqs[0, 0, 2] < 2.0 ** -126 or dtype == "fp16"


def test_quantiser_q_only_and_k_only_calls():
    w = small(GQA, D=128, Lq=300, Lk=520, B=1, H=4, Hkv=2)
    t = make_workload(w)
    q, k = to_dev(t.q_bits, w.dtype), to_dev(t.k_bits, w.dtype)
    q8 = torch.zeros(q.shape, device="cuda", dtype=torch.uint8)
    k8 = torch.zeros(k.shape, device="cuda", dtype=torch.uint8)
    qs = torch.zeros((1, 4, 3), device="cuda", dtype=torch.float32)
    ks = torch.zeros((1, 2, 5), device="cuda", dtype=torch.float32)
    mode = mpt.mode_bits(fmt="int8", dtype=w.dtype)
    mpt.lamp_quant_qk(q, None, q8, None, qs, None, 1, 4, 2, 300, 520, 128, mode)
    torch.cuda.synchronize()
    assert int(k8.count_nonzero()) == 0 and int(ks.count_nonzero()) == 0
    mpt.lamp_quant_qk(None, k, None, k8, None, ks, 1, 4, 2, 300, 520, 128, mode)
    torch.cuda.synchronize()
    rq, rqs = oracle.quantize(t.q, 128, "int8")
    rk, rks = oracle.quantize(t.k, 128, "int8")
    assert np.array_equal(q8.cpu().numpy(), rq) and np.array_equal(qs.cpu().numpy(), rqs)
    assert np.array_equal(k8.cpu().numpy(), rk) and np.array_equal(ks.cpu().numpy(), rks)


@pytest.mark.parametrize("B,H,L,D,g,p", [(1, 1, 256, 64, 1, 0.25), (2, 32, 4096, 128, 4, 0.2),
                                         (1, 32, 131072, 128, 8, 0.1), (1, 8, 16384, 256, 2, 0.3),
                                         (1, 2, 8193, 128, 1, 0.5)])
def test_mask_builder_bit_exact(B, H, L, D, g, p):
    bm, bn = mpt.lamp_tile_shape(D)
    m = mpt.build_mask(B, H, L, L, D, g, p, 1234)
    torch.cuda.synchronize()
    nqt, nkt = -(-L // bm), -(-L // bn)
    ref = oracle.build_mask(B, H, nqt, nkt, g, p, 1234)
    assert np.array_equal(mask_to_numpy(m), ref)


@pytest.mark.parametrize("B,H,Lq,Lk,D,g,sink,band,stride", [
    (1, 1, 512, 512, 64, 1, 1, 2, 3), (2, 3, 4096, 4096, 128, 4, 0, 1, 4),
    (1, 2, 200, 300, 64, 2, 0, 1, 2), (1, 2, 700, 300, 128, 1, 2, 1, 0),
    (1, 4, 16384, 16384, 256, 2, 1, 1, 4), (1, 1, 130 * 128, 130 * 128, 128, 1, 1, 3, 7)])
def test_mask_template_bit_exact(B, H, Lq, Lk, D, g, sink, band, stride):
    bm, bn = mpt.lamp_tile_shape(D)
    m = mpt.build_mask_template(B, H, Lq, Lk, D, g, sink, band, stride)
    torch.cuda.synchronize()
    ref = oracle.build_mask_template(B, H, Lq, Lk, bm, bn, g, sink, band, stride)
    assert np.array_equal(mask_to_numpy(m), ref)


def test_attention_with_sptrans75_template():
    # the 75%-INT8 structured template chosen by the library's search, end to end against the
    # oracle on the same mask (GQA, causal, ragged tail)
    w = CONFIGS["gqa4k"].replace(H=4, Hkv=2, Lq=1000, Lk=1000)
    sink, band, stride, fr = mpt.lamp_template_for_int8_fraction(w.Lq, w.Lk, w.D, w.group_tiles,
                                                                  1, 0, 0.75)
    t = make_workload(w)
    mask_dev = mpt.build_mask_template(w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles, sink, band,
                                       stride)
    mask = mask_to_numpy(mask_dev)
    g = gpu_run(w, t, mask_dev=mask_dev)
    r = oracle_run(w, t, mask=mask)
    assert np.array_equal(g["route"], r["route"])
    live = g["route"] > 0
    assert 0 < (g["route"][live] == 2).mean() < 1
    check_outputs(g, r, what="sptrans75")


# ----------------------------------------------------------------- attention, small ----

def test_tiny_workload():
    parity_case(TINY)


@pytest.mark.parametrize("p", [0.0, 0.3, 1.0])
def test_d128_causal_gqa_ragged(p):
    w = small(GQA, B=2, H=4, Hkv=2, Lq=600, Lk=600, group_tiles=2)
    parity_case(w, p_fp16=p)


def test_d128_noncausal_ragged_both():
    w = small(GQA, B=1, H=2, Hkv=1, Lq=300, Lk=520, causal=False, group_tiles=1)
    parity_case(w, p_fp16=0.4)


@pytest.mark.parametrize("Lq,Lk", [(200, 700), (700, 200)])
def test_d128_causal_bottom_right(Lq, Lk):
    w = small(GQA, B=1, H=2, Hkv=2, Lq=Lq, Lk=Lk, group_tiles=1, plant_frac=0.0)
    parity_case(w, p_fp16=0.5)


@pytest.mark.parametrize("dtype,p", [("fp16", 0.5), ("bf16", 0.5), ("bf16", 0.0)])
def test_d64_stacked_tiles(dtype, p):
    w = small(TINY, B=1, H=2, Hkv=1, Lq=320, Lk=320, causal=True, dtype=dtype, values="structured",
              plant_frac=0.02)
    parity_case(w, p_fp16=p)


@pytest.mark.parametrize("window", [0, 200])
def test_d256_stacked_window(window):
    w = small(CONFIGS["gemma_local16k"], B=1, H=4, Hkv=2, Lq=700, Lk=700, window=window)
    parity_case(w)


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
def test_all_8bit_and_e4m3_bitmask(fmt):
    w = small(GQA, B=1, H=2, Hkv=1, Lq=512, Lk=512)
    parity_case(w, none8=True, fmt=fmt)
    parity_case(w, p_fp16=0.3, fmt=fmt)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_all_16bit_routing_is_exact_attention(dtype):
    w = small(GQA, B=1, H=2, Hkv=1, Lq=384, Lk=384, dtype=dtype, values="iid", plant_frac=0.0)
    g, r = parity_case(w, all16=True)
    err = np.abs(g["o"] - r["o"]).max()
    assert err <= EXACT_MAX_ABS, err


def test_v_ones_gives_ones():
    for w, kw in [(small(GQA, B=1, H=2, Hkv=1, Lq=400, Lk=400), dict(p_fp16=0.3)),
                  (small(CONFIGS["adaptive8k"], B=1, H=2, Hkv=1, Lq=400, Lk=400), {}),
                  (small(TINY, Lq=200, Lk=200, causal=True), dict(p_fp16=0.5))]:
        g, _ = parity_case(w, v_ones=True, **kw)
        assert np.abs(g["o"][np.isfinite(g["lse"])] - 1.0).max() < 1e-5


def test_output_in_input_dtype():
    w = small(GQA, B=1, H=2, Hkv=1, Lq=256, Lk=256)
    g, r = parity_case(w, p_fp16=0.3, out="in")
    assert np.abs(g["o"] - r["o"]).max() < 2e-2


def test_output_in_input_dtype_d256_ragged():
    # D = 256 writes O through a shared-memory staging area: 16-bit output, a ragged last
    # query tile (rows past Lq must not be written) and a sliding window
    w = small(CONFIGS["gemma_local16k"], B=1, H=2, Hkv=1, Lq=333, Lk=333, window=200)
    g, r = parity_case(w, p_fp16=0.3, out="in")
    assert np.abs(g["o"] - r["o"]).max() < 2e-2


@pytest.mark.parametrize("fmt", ["int8", "e4m3"])
@pytest.mark.parametrize("tau", [-1e30, 2.0, 4.0, 8.0])
def test_adaptive_small(fmt, tau):
    w = small(CONFIGS["adaptive8k"], B=1, H=4, Hkv=2, Lq=768, Lk=768)
    g, r = parity_case(w, fmt=fmt, tau=tau)
    live = g["route"] != 0
    assert set(np.unique(g["route"][live]).tolist()) <= {1, 3}
    if tau < 0:  # only tiles holding a row's first visible key can be flagged
        assert np.all(g["route"][..., 0] == 3)
        assert np.all(g["route"][..., 1:][live[..., 1:]] == 1)


@pytest.mark.parametrize("base", ["tiny", "gemma_local16k"])
def test_adaptive_stacked(base):
    b = CONFIGS[base]
    w = small(b, B=1, H=2, Hkv=1, Lq=330, Lk=330, causal=True, route="adaptive", tau=3.0,
              values="structured", plant_frac=0.02, window=0)
    parity_case(w, fmt="int8", tau=3.0)


# ----------------------------------------------------------------- threshold skip -----

@pytest.mark.parametrize("D,fmt,window,L", [(128, "int8", 0, 1100), (128, "e4m3", 0, 700),
                                            (64, "int8", 0, 600), (256, "int8", 300, 900)])
def test_threshold_skip_matches_oracle(D, fmt, window, L):
    # look-ahead routing with a threshold skip: decisions (within the 1e-3 margin), codes and
    # outputs against the oracle; the skip must actually drop tiles here
    bm, bn = mpt.lamp_tile_shape(D)
    w = small(CONFIGS["adaptive8k"], B=1, H=2, Hkv=1, Lq=L, Lk=L, D=D, bm=bm, bn=bn,
              window=window, fmt=fmt, tau=2.0)
    skip = 6.0
    # inputs whose key tiles sit at seeded offsets along a direction every query shares, so
    # that whole tiles fall far below the running max (the workload generators rarely do)
    rng = np.random.default_rng(17)
    u = rng.standard_normal(D)
    u *= 0.5 * np.sqrt(D) / np.linalg.norm(u)
    qf = rng.standard_normal((1, 2, L, D)) + 3.0 * u
    shift = np.repeat(rng.choice([1.0, 0.0, -1.0, -2.0], size=-(-L // bn)), bn)[:L]
    kf = rng.standard_normal((1, 1, L, D)) + shift[None, None, :, None] * u
    vf = rng.standard_normal((1, 1, L, D))
    q, k, v = (torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda()
               for x in (qf, kf, vf))
    t = type("T", (), {})()
    t.q, t.k, t.v = (x.float().cpu().numpy() for x in (q, k, v))
    q8, k8, qs, ks = mpt.quantize(q, k, fmt=fmt)
    o, lse, rmap = mpt.attention_q8(q, k, v, q8, k8, qs, ks, causal=True, window=window,
                                    route="adaptive", fmt=fmt, tau=w.tau, skip_tau=skip,
                                    want_route=True)
    torch.cuda.synchronize()
    mpt.lamp_check()
    g = {"o": o.cpu().numpy().astype(np.float64), "lse": lse.cpu().numpy().astype(np.float64),
         "route": rmap.cpu().numpy()}
    r = oracle.attention(t.q, t.k, t.v, bm=bm, bn=bn, causal=True, window=window,
                         route="adaptive", fmt=fmt, tau=w.tau, skip_tau=skip,
                         route_hint=g["route"], hint_margin=1e-3)
    assert np.array_equal(g["route"], r["route"])
    assert (g["route"] == 4).any() and (g["route"] == 3).any()
    check_outputs(g, r, what=f"skip D={D} {fmt}")


def test_threshold_skip_infinite_is_the_look_ahead_rule():
    w = small(CONFIGS["adaptive8k"], B=1, H=2, Hkv=1, Lq=600, Lk=600, fmt="e4m3", tau=3.0)
    t = make_workload(w)
    q, k, v = (to_dev(x, w.dtype) for x in (t.q_bits, t.k_bits, t.v_bits))
    q8, k8, qs, ks = mpt.quantize(q, k, fmt="e4m3")
    kw = dict(causal=True, route="adaptive", fmt="e4m3", tau=3.0, want_route=True)
    a = mpt.attention_q8(q, k, v, q8, k8, qs, ks, **kw)
    b = mpt.attention_q8(q, k, v, q8, k8, qs, ks, skip_tau=float("inf"), **kw)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ----------------------------------------------------------------- full size, sampled --

@pytest.mark.parametrize("name", ["gqa4k", "gemma_local16k"])
def test_full_size_bitmask_whole_output(name):
    # every row of the full workload against the oracle (about 2 s of oracle time each)
    parity_case(CONFIGS[name], check_codes=False)


@pytest.mark.parametrize("name", ["long32k", "long64k", "long128k"])
def test_full_size_bitmask_sampled_rows(name):
    w = CONFIGS[name]
    rows = sample_rows(w, 64)
    parity_case(w, rows=rows, check_codes=False)


def test_masks_wider_than_two_words_sampled_rows():
    # 129 key groups (three mask words) at D = 128: the bits past group 127 must be honoured
    w = CONFIGS["gqa4k"].replace(B=1, H=2, Hkv=1, Lq=129 * 128, Lk=129 * 128, group_tiles=1,
                                 p_fp16=0.5)
    assert mpt.lamp_mask_words(w.Lk, w.D, w.group_tiles) == 3
    tail = np.array([w.Lq - 128, w.Lq - 64, w.Lq - 1])  # rows of the last query tile see group 128
    one = np.union1d(np.linspace(0, w.Lq - 1, 45).astype(np.int64), tail)
    rows = np.broadcast_to(one, (w.B, w.H, one.size)).copy()
    parity_case(w, rows=rows, check_codes=False)


@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
@pytest.mark.parametrize("tau", [2.0, 4.0, 8.0])
def test_full_size_adaptive_sampled_tiles(fmt, tau):
    # adaptive8k at full size in the benchmark's launch configuration: INT8 runs on the
    # persistent two-tile kernel (2048 work items over one CTA per SM, so every CTA walks many
    # items and the next item's start overlaps the current one's tail), E4M3 on the single-tile
    # kernel; whole query tiles (a tile's decisions depend on all its rows), one per head
    w = CONFIGS["adaptive8k"]
    tiles = sample_tiles(w, 1, seed=int(tau) + (10 if fmt == "int8" else 0))
    rows = (tiles[..., None] * w.bm + np.arange(w.bm)[None, None, None, :]).reshape(w.B, w.H, -1)
    parity_case(w, rows=rows, fmt=fmt, tau=tau, check_codes=False)


# ----------------------------------------------------------------- failure path -------

def test_bounded_wait_reports_timeout():
    mpt.lamp_selftest_timeout(1_000_000)  # 1 ms on a barrier nothing completes
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_check()
    assert e.value.code == mpt.LAMP_ERR_TIMEOUT
    mpt.lamp_check()  # the error word was cleared; the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def test_mma_probe_runs():
    for kind in (0, 1, 2):
        for n in (64, 128, 256):
            mpt.lamp_mma_probe(kind, n, 8)
    torch.cuda.synchronize()
    mpt.lamp_check()
