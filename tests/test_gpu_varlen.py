"""Variable-length batches (TileMix page, section 4: GQA and variable-length batches are
supported) on the GPU, through the C ABI.

Sequences of a variable-length batch are independent problems, so the oracle is the dense
oracle run once per sequence on that sequence's rows; the mask is the padded [B][H][nQT][W]
layout.  Also checked: a batch of equal-length sequences gives bit-for-bit the outputs of the
dense call on the same data."""
import types

import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
import oracle
from workloads import CONFIGS, make_workload

from _parity import check_outputs, mask_to_numpy, to_dev

pytestmark = pytest.mark.gpu


def make_batch(base, lq, lk, seed0=500):
    """Per-sequence seeded data packed head-major: q [H][total_q][D], k, v [Hkv][total_k][D]."""
    seqs = []
    for i, (a, b) in enumerate(zip(lq, lk)):
        if a and b:
            seqs.append(make_workload(base.replace(B=1, Lq=a, Lk=b, seed=seed0 + i)))
        else:  # an empty sequence: no rows of its own in the packed tensors
            z = lambda n, h: np.zeros((1, h, n, base.D), dtype=np.uint16)
            seqs.append(types.SimpleNamespace(q_bits=z(a, base.H), k_bits=z(b, base.Hkv),
                                              v_bits=z(b, base.Hkv)))
    q = np.concatenate([t.q_bits[0] for t in seqs], axis=1)
    k = np.concatenate([t.k_bits[0] for t in seqs], axis=1)
    v = np.concatenate([t.v_bits[0] for t in seqs], axis=1)
    return seqs, q, k, v


def run_varlen(base, lq, lk, *, route="bitmask", fmt="int8", p_fp16=0.3, tau=4.0, seed0=500):
    w = base
    B = len(lq)
    max_q, max_k = max(max(lq), 1), max(max(lk), 1)
    seqs, qb, kb, vb = make_batch(base, lq, lk, seed0)
    q, k, v = (to_dev(x, w.dtype) for x in (qb, kb, vb))
    tq, tk = q.shape[1], k.shape[1]
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    bm, bn = mpt.lamp_tile_shape(w.D)
    nqt, nkt = -(-max_q // bm), -(-max_k // bn)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
    qs = torch.full((B, w.H, nqt), -1.0, device="cuda")
    ks = torch.full((B, w.Hkv, nkt), -1.0, device="cuda")
    mode = mpt.mode_bits(route, fmt, w.dtype)
    mpt.lamp_quant_qk_varlen(q, k, q8, k8, qs, ks, cu_q, cu_k, B, w.H, w.Hkv, max_q, max_k, tq,
                             tk, w.D, mode)
    mask = None
    if route == "bitmask":
        mask = mpt.build_mask(B, w.H, max_q, max_k, w.D, w.group_tiles, p_fp16, 77)
    o = torch.full((w.H, tq, w.D), float("nan"), device="cuda")
    lse = torch.full((w.H, tq), float("nan"), device="cuda")
    rmap = torch.empty((B, w.H, nqt, nkt), dtype=torch.uint8, device="cuda")
    mpt.lamp_attn_fwd_q8_varlen(q, k, v, q8, k8, qs, ks, o, lse, cu_q, cu_k, B, w.H, w.Hkv,
                                max_q, max_k, tq, tk, w.D, w.causal, w.window, 0.0, mask,
                                w.group_tiles, mode, tau, rmap)
    torch.cuda.synchronize()
    mpt.lamp_check()
    return dict(seqs=seqs, cu_q=cu_q.cpu().numpy(), cu_k=cu_k.cpu().numpy(), o=o.cpu().numpy(),
                lse=lse.cpu().numpy(), q8=q8.cpu().numpy(), k8=k8.cpu().numpy(),
                qs=qs.cpu().numpy(), ks=ks.cpu().numpy(), route=rmap.cpu().numpy(),
                mask=mask_to_numpy(mask) if mask is not None else None, bm=bm, bn=bn)


def check_against_oracle(base, lq, lk, g, *, route="bitmask", fmt="int8", tau=4.0):
    w = base
    for b, t in enumerate(g["seqs"]):
        a, c = lq[b], lk[b]
        q0, k0 = g["cu_q"][b], g["cu_k"][b]
        nqt_b, nkt_b = -(-a // g["bm"]), -(-c // g["bn"])
        if a == 0 or c == 0:
            continue
        m = None if g["mask"] is None else np.ascontiguousarray(g["mask"][b:b + 1, :, :nqt_b])
        hint = g["route"][b:b + 1, :, :nqt_b, :nkt_b] if route == "adaptive" else None
        r = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, causal=w.causal, window=w.window,
                             mask=m, group_tiles=w.group_tiles, route=route, fmt=fmt, tau=tau,
                             want_codes=True, route_hint=hint,
                             hint_margin=1e-3 if hint is not None else 0.0)
        # codes and scales of this sequence's rows and blocks, bit-exact
        assert np.array_equal(g["q8"][:, q0:q0 + a], r["q_codes"][0]), ("q codes", b)
        if c:
            assert np.array_equal(g["k8"][:, k0:k0 + c], r["k_codes"][0]), ("k codes", b)
            assert np.array_equal(g["ks"][b, :, :nkt_b], r["k_scales"][0]), ("k scales", b)
        assert np.array_equal(g["qs"][b, :, :nqt_b], r["q_scales"][0]), ("q scales", b)
        assert np.array_equal(g["route"][b, :, :nqt_b, :nkt_b], r["route"][0]), ("route", b)
        got = {"o": g["o"][None, :, q0:q0 + a].astype(np.float64),
               "lse": g["lse"][None, :, q0:q0 + a].astype(np.float64)}
        check_outputs(got, r, what=f"{w.name} sequence {b}")


CASES = [
    # (workload, query lengths, key lengths)
    ("gqa4k", [300, 0, 1000, 129, 640], None),          # two-tile kernel, empty sequence
    ("gqa4k", [256, 700], [600, 900]),                    # more keys than queries per sequence
    ("tiny", [64, 250, 1, 513], None),                    # D = 64, stacked 64-row tiles
    ("gemma_local16k", [1500, 700, 2100], None),          # D = 256 with the sliding window
]


@pytest.mark.parametrize("name,lq,lk", CASES)
def test_varlen_bitmask_matches_per_sequence_oracle(name, lq, lk):
    base = CONFIGS[name].replace(H=min(CONFIGS[name].H, 4), Hkv=min(CONFIGS[name].Hkv, 2))
    lk = lq if lk is None else lk
    g = run_varlen(base, lq, lk)
    check_against_oracle(base, lq, lk, g)


@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
def test_varlen_adaptive_matches_per_sequence_oracle(fmt):
    base = CONFIGS["adaptive8k"].replace(H=2, Hkv=1)
    lq = [200, 520, 77]
    g = run_varlen(base, lq, lq, route="adaptive", fmt=fmt, tau=4.0)
    check_against_oracle(base, lq, lq, g, route="adaptive", fmt=fmt, tau=4.0)


@pytest.mark.parametrize("name", ["gqa4k", "tiny", "gemma_local16k"])
def test_equal_lengths_match_the_dense_call_bitwise(name):
    # B sequences of one length: the packed call and the dense [B][H][L][D] call see the same
    # data and must give identical bits
    base = CONFIGS[name].replace(H=min(CONFIGS[name].H, 4), Hkv=min(CONFIGS[name].Hkv, 2))
    L, B = 640, 3
    g = run_varlen(base, [L] * B, [L] * B)
    w = base.replace(B=B, Lq=L, Lk=L)
    dense_q = np.stack([t.q_bits[0] for t in g["seqs"]])
    dense_k = np.stack([t.k_bits[0] for t in g["seqs"]])
    dense_v = np.stack([t.v_bits[0] for t in g["seqs"]])
    q, k, v = (to_dev(x, w.dtype) for x in (dense_q, dense_k, dense_v))
    q8, k8, qs, ks = mpt.quantize(q, k, fmt="int8")
    mask = mpt.build_mask(B, w.H, L, L, w.D, w.group_tiles, 0.3, 77)
    o, lse, _ = mpt.attention_q8(q, k, v, q8, k8, qs, ks, causal=w.causal, window=w.window,
                                 mask_bits=mask, group_tiles=w.group_tiles, want_route=True)
    torch.cuda.synchronize()
    o_d = o.cpu().numpy().transpose(1, 0, 2, 3).reshape(w.H, B * L, w.D)
    lse_d = lse.cpu().numpy().transpose(1, 0, 2).reshape(w.H, B * L)
    assert np.array_equal(g["o"], o_d)
    assert np.array_equal(g["lse"], lse_d, equal_nan=True)
