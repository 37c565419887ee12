"""8-bit exponentials and an 8-bit P.V against the oracle (GPU).

Reading (LampAttention abstract: exponentials in 8-bit formats; the pages fix no format): V in
E4M3 with one scale per (batch, KV head, channel) over all keys; each p = 2^(x - m_t) * 2^8
rounded to E4M3 against the running max after its key tile; O = v_scale * sum p8 v8 / sum p8;
lse of the exact p.  Checks:
  * the V quantiser (codes, padding, scales) bit-exact against ``oracle.quantize_v``;
  * O against ``oracle.attention(pv8=True)``: the GPU's scores and running max are fp32, the
    oracle's fp64 (about 1e-6 relative apart), so a p within that distance of an E4M3 rounding
    midpoint may round either way.  Rows whose every p is at least 1e-5 (relative) from a
    midpoint (the oracle's ``pv8_margin``) must match to fp32 accumulation accuracy, 2e-4 of
    max |V|; the other rows within the bound of rounding flips, and they stay a minority;
  * lse within 1e-3 of the oracle's (exact p); the end-to-end call and the kernel alone on
    separately quantised operands bit-identical.
"""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt
import oracle

pytestmark = pytest.mark.gpu

MARGIN = 1e-5


def _inputs(B, H, Hkv, Lq, Lk, D, dt, seed, v_zero_channel=False):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, H, Lq, D), generator=g).to(dt)
    k = torch.randn((B, Hkv, Lk, D), generator=g).to(dt)
    v = torch.randn((B, Hkv, Lk, D), generator=g).to(dt)
    if v_zero_channel:
        v[..., 5] = 0
    return q, k, v


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_v_quantiser_bit_exact(D, dt):
    B, Hkv, Lk = 2, 3, 300  # keys not a multiple of 16: padded rows
    _, _, v = _inputs(B, 1, Hkv, 1, Lk, D, dt, seed=D, v_zero_channel=True)
    v8t, vs = mpt.quantize_v(v.cuda())
    torch.cuda.synchronize()
    mpt.lamp_check()
    codes, scales = oracle.quantize_v(v.float().numpy())
    g8 = v8t.cpu().numpy()
    assert g8.shape == (B, Hkv, D, 304)
    assert np.array_equal(g8[..., :Lk], codes)
    assert np.all(g8[..., Lk:] == 0)
    assert np.array_equal(vs.cpu().numpy(), scales)


CASES = [
    # B, H, Hkv, Lq, Lk, causal, window, route, fmt, p16, tau, dtype
    (1, 4, 2, 700, 700, True, 0, "bitmask", "int8", 0.3, 0.0, torch.bfloat16),
    (2, 2, 1, 520, 520, True, 0, "adaptive", "e4m3", 0.0, 4.0, torch.bfloat16),
    (1, 2, 2, 300, 900, False, 0, "bitmask", "int8", 0.0, 0.0, torch.float16),
    (1, 2, 1, 1000, 1000, True, 300, "bitmask", "int8", 0.5, 0.0, torch.bfloat16),
    (1, 2, 2, 640, 640, True, 0, "bitmask", "e4m3", 1.0, 0.0, torch.bfloat16),
]


@pytest.mark.parametrize("B,H,Hkv,Lq,Lk,causal,window,route,fmt,p16,tau,dt", CASES)
def test_pv8_attention_matches_oracle(B, H, Hkv, Lq, Lk, causal, window, route, fmt, p16, tau, dt):
    D, g = 128, 2
    q, k, v = _inputs(B, H, Hkv, Lq, Lk, D, dt, seed=Lq + Lk + H)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    mask = mpt.build_mask(B, H, Lq, Lk, D, g, p16, 11) if route == "bitmask" else None
    kw = dict(causal=causal, window=window, mask_bits=mask, group_tiles=g, route=route, fmt=fmt,
              tau=tau)
    o, lse = mpt.attention(dq, dk, dv, pv8=True, **kw)
    # the kernel alone on separately quantised operands: the same bits
    q8, k8, qs, ks = mpt.quantize(dq, dk, fmt=fmt)
    v8t, vs = mpt.quantize_v(dv)
    o2, lse2 = mpt.attention_q8_pv8(dq, dk, q8, k8, qs, ks, v8t, vs, **kw)
    # the route map of the 16-bit P kernel: the look-ahead decisions do not depend on P's format
    _, _, rmap = mpt.attention_q8(dq, dk, dv, q8, k8, qs, ks, want_route=True, **kw)
    torch.cuda.synchronize()
    mpt.lamp_check()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    ref = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), bm=128, bn=128,
                           causal=causal, window=window,
                           mask=None if mask is None else mask.cpu().numpy().view(np.uint64),
                           group_tiles=g, route=route, fmt=fmt, tau=tau, pv8=True,
                           route_hint=rmap.cpu().numpy(), hint_margin=1e-3)
    assert ref["hinted"].sum() <= max(1, int(0.001 * (ref["route"] > 0).sum()))
    go, gl = o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    vmax = float(np.abs(v.float().numpy()).max())
    err = np.abs(go - ref["o"]).max(axis=-1)                      # [B, H, Lq]
    sure = ref["pv8_margin"] >= MARGIN
    assert sure.mean() > 0.7, sure.mean()
    assert err[sure].max() <= 2e-4 * vmax, (err[sure].max(), vmax)
    assert err[~sure].max(initial=0.0) <= 0.25 * vmax
    fin = np.isfinite(ref["lse"])
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - ref["lse"][fin]).max() <= 1e-3
    # and within the E4M3 rounding bound of the 16-bit P result on the same inputs
    o16, _ = mpt.attention(dq, dk, dv, **kw)
    assert (o16 - o).abs().max().item() <= 2 * 2.0 ** -4 * vmax


def test_pv8_through_the_allocation_free_and_host_buffer_entries():
    # both quantise V themselves in this mode: bit-identical to lamp_attn_fwd
    B, H, Hkv, L, D = 2, 4, 2, 600, 128
    q, k, v = _inputs(B, H, Hkv, L, L, D, torch.bfloat16, seed=3)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    mask = mpt.build_mask(B, H, L, L, D, 2, 0.3, 5)
    mode = mpt.mode_bits("bitmask", "int8", "bf16", pv8=True)
    o = torch.empty((B, H, L, D), device="cuda", dtype=torch.float32)
    lse = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
    mpt.lamp_attn_fwd(dq, dk, dv, o, lse, B, H, Hkv, L, L, D, 1, 0, 0.0, mask, 2, mode, 0.0)
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    mpt.lamp_attn_fwd_noalloc(dq, dk, dv, o2, lse2, B, H, Hkv, L, L, D, 1, 0, 0.0, mask, 2, mode,
                              0.0)
    hin = [x.pin_memory() for x in (q, k, v)]
    ho = torch.empty((B, H, L, D), dtype=torch.float32).pin_memory()
    hl = torch.empty((B, H, L), dtype=torch.float32).pin_memory()
    mpt.lamp_attn_fwd_host(*hin, ho, hl, B, H, Hkv, L, L, D, 1, 0, 0.0, mask, 2, mode, 0.0,
                           n_chunks=3)
    torch.cuda.synchronize()
    mpt.lamp_check()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(ho, o.cpu()) and torch.equal(hl, lse.cpu())


@pytest.mark.parametrize("out", ["f32", "in"])
def test_pv8_full_size_gqa4k_sampled_rows(out):
    # the gqa4k workload's shape and inputs (B=1 H=32 Hkv=8 L=4096, INT8, structured values) in
    # the 8-bit P.V mode, 64 seeded rows per head against the oracle; O in fp32 and in bf16.
    # Every tile 8-bit: the scores are exact integers times one fp32 constant on both sides, so
    # the GPU's p stays within ~1e-6 of the oracle's and the 1e-5 midpoint margin holds for
    # 4096-key rows (16-bit tiles, whose fp32 tensor-core sums add their own error, are covered
    # by the smaller cases above)
    from workloads import CONFIGS, make_workload, sample_rows
    w = CONFIGS["gqa4k"].replace(p_fp16=0.0)
    t = make_workload(w)
    dq, dk, dv = (torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
                  for b in (t.q_bits, t.k_bits, t.v_bits))
    mask = mpt.build_mask(w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles, w.p_fp16, w.mask_seed)
    o, lse = mpt.attention(dq, dk, dv, causal=True, mask_bits=mask, group_tiles=w.group_tiles,
                           fmt=w.fmt, out=out, pv8=True)
    torch.cuda.synchronize()
    mpt.lamp_check()
    rows = sample_rows(w, 64, seed=21)
    ref = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, causal=True,
                           mask=mask.cpu().numpy().view(np.uint64), group_tiles=w.group_tiles,
                           fmt=w.fmt, rows=rows, pv8=True)
    go = o.float().cpu().numpy().astype(np.float64)
    gl = lse.cpu().numpy().astype(np.float64)
    go = np.stack([np.stack([go[0, h, rows[0, h]] for h in range(w.H)])])
    gl = np.stack([np.stack([gl[0, h, rows[0, h]] for h in range(w.H)])])
    vmax = float(np.abs(t.v).max())
    # bf16 output adds its own rounding: half an ulp of |O| <= vmax
    tol = 2e-4 * vmax + (0.0 if out == "f32" else vmax * 2.0 ** -8)
    err = np.abs(go - ref["o"]).max(axis=-1)
    sure = ref["pv8_margin"] >= MARGIN
    assert sure.mean() > 0.5, sure.mean()
    assert err[sure].max() <= tol, (err[sure].max(), tol)
    assert err[~sure].max(initial=0.0) <= 0.25 * vmax
    assert np.abs(gl - ref["lse"]).max() <= 1e-3
