"""Shared helpers of the GPU parity tests: run one workload through the CUDA library and
through the CPU oracle on the same seeded inputs, and compare with the acceptance tolerances.

Tolerances (stated with the workload definitions of this build):
  * quantised codes, scales, routing decisions: bit-exact (adaptive decisions whose oracle
    margin is below ADAPTIVE_MARGIN may differ; the oracle then follows the GPU's decision and
    everything downstream is compared against that re-run);
  * O: max-abs <= O_MAX_ABS and mean-abs <= O_MEAN_ABS against the oracle (unit-variance V);
  * lse: abs <= LSE_ABS;
  * all-16-bit routing against exact fp64 attention: max-abs <= EXACT_MAX_ABS.
Look-ahead cases also bound how many decisions the oracle took from the GPU's route map:
HINTED_MAX of the live tiles (at least one), each with an oracle margin below ADAPTIVE_MARGIN.
"""
import numpy as np
import torch

import mixed_precision_tiled_b200 as mpt
import oracle
from workloads import make_workload

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 1e-3
EXACT_MAX_ABS = 4e-3
ADAPTIVE_MARGIN = 1e-3
HINTED_MAX = 1e-3


def to_dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16).cuda()


def mask_to_numpy(m: torch.Tensor) -> np.ndarray:
    return m.cpu().numpy().view(np.uint64)


def gpu_run(w, t, *, mask_dev=None, route=None, fmt=None, tau=None, out="f32"):
    route = route or w.route
    fmt = fmt or w.fmt
    tau = w.tau if tau is None else tau
    q, k, v = (to_dev(x, w.dtype) for x in (t.q_bits, t.k_bits, t.v_bits))
    q8, k8, qs, ks = mpt.quantize(q, k, fmt=fmt)
    o, lse, rmap = mpt.attention_q8(q, k, v, q8, k8, qs, ks, causal=w.causal, window=w.window,
                                    mask_bits=mask_dev, group_tiles=w.group_tiles, route=route,
                                    fmt=fmt, tau=tau, out=out, want_route=True)
    torch.cuda.synchronize()
    mpt.lamp_check()
    return {
        "o": o.float().cpu().numpy().astype(np.float64),
        "lse": lse.cpu().numpy().astype(np.float64),
        "route": rmap.cpu().numpy(),
        "q8": q8.cpu().numpy(), "k8": k8.cpu().numpy(),
        "qs": qs.cpu().numpy(), "ks": ks.cpu().numpy(),
    }


def gpu_mask(w, p_fp16=None, seed=None):
    p = w.p_fp16 if p_fp16 is None else p_fp16
    return mpt.build_mask(w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles, p,
                          w.mask_seed if seed is None else seed)


def check_outputs(g, r, *, rows=None, o_max=O_MAX_ABS, o_mean=O_MEAN_ABS, lse_abs=LSE_ABS,
                  what=""):
    o_g, lse_g = g["o"], g["lse"]
    if rows is not None:
        B, H, _ = rows.shape
        o_g = np.stack([np.stack([o_g[b, h, rows[b, h]] for h in range(H)]) for b in range(B)])
        lse_g = np.stack([np.stack([lse_g[b, h, rows[b, h]] for h in range(H)]) for b in range(B)])
    fin = np.isfinite(r["lse"])
    assert np.array_equal(fin, np.isfinite(lse_g)), f"{what}: empty-row pattern differs"
    assert np.all(o_g[~fin] == 0.0), f"{what}: rows without keys must be 0"
    err = np.abs(o_g - r["o"])
    assert np.isfinite(o_g).all(), f"{what}: non-finite O"
    mx, mean = err.max(), err.mean()
    lerr = np.abs(lse_g[fin] - r["lse"][fin]).max() if fin.any() else 0.0
    assert mx <= o_max, f"{what}: O max-abs {mx:.3e} > {o_max}"
    assert mean <= o_mean, f"{what}: O mean-abs {mean:.3e} > {o_mean}"
    assert lerr <= lse_abs, f"{what}: lse abs {lerr:.3e} > {lse_abs}"
    return mx, mean, lerr


def oracle_run(w, t, *, mask=None, route=None, fmt=None, tau=None, rows=None, hint=None,
               want_codes=False):
    return oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, causal=w.causal, window=w.window,
                            mask=mask, group_tiles=w.group_tiles, route=route or w.route,
                            fmt=fmt or w.fmt, tau=w.tau if tau is None else tau, rows=rows,
                            route_hint=hint, hint_margin=ADAPTIVE_MARGIN if hint is not None else 0.0,
                            want_codes=want_codes)


def parity_case(w, *, p_fp16=None, route=None, fmt=None, tau=None, all16=False, none8=False,
                v_ones=False, rows=None, out="f32", check_codes=True):
    """Runs one case on both sides; returns (gpu, oracle) results after all checks."""
    route = route or w.route
    fmt = fmt or w.fmt
    t = make_workload(w, v_ones=v_ones)
    mask_dev, mask = None, None
    if route == "bitmask" and not none8:
        mask_dev = gpu_mask(w, 1.0 if all16 else p_fp16)
        mask = mask_to_numpy(mask_dev)
        ref_mask = oracle.build_mask(w.B, w.H, w.nqt, w.nkt, w.group_tiles,
                                     1.0 if all16 else (w.p_fp16 if p_fp16 is None else p_fp16),
                                     w.mask_seed)
        assert np.array_equal(mask, ref_mask), "mask builder differs from the oracle"
    g = gpu_run(w, t, mask_dev=mask_dev, route=route, fmt=fmt, tau=tau, out=out)
    hint = g["route"] if route == "adaptive" else None
    r = oracle_run(w, t, mask=mask, route=route, fmt=fmt, tau=tau, rows=rows, hint=hint,
                   want_codes=check_codes)
    if check_codes:
        assert np.array_equal(g["q8"], r["q_codes"]), "Q codes differ"
        assert np.array_equal(g["k8"], r["k_codes"]), "K codes differ"
        assert np.array_equal(g["qs"], r["q_scales"]), "Q scales differ"
        assert np.array_equal(g["ks"], r["k_scales"]), "K scales differ"
    if route == "adaptive":
        # decisions the oracle took from the GPU's map instead of its own outcome: few, and
        # each within the margin where two correct implementations may disagree
        hinted = r["hinted"].astype(bool)
        live = int((r["route"] > 0).sum())
        assert int(hinted.sum()) <= max(1, HINTED_MAX * live), (int(hinted.sum()), live)
        assert np.all(r["margin"][hinted] < ADAPTIVE_MARGIN)
    if rows is None:
        assert np.array_equal(g["route"], r["route"]), "routing map differs"
    else:
        # only the query tiles that hold sampled rows were routed by the oracle
        B, H, _ = rows.shape
        for b in range(B):
            for h in range(H):
                for qt in np.unique(rows[b, h] // w.bm):
                    assert np.array_equal(g["route"][b, h, qt], r["route"][b, h, qt]), (b, h, qt)
    if out == "f32":
        check_outputs(g, r, rows=rows, what=w.name)
    else:  # O rounded to the 16-bit input type: half an ulp of bf16 at |O| < 4 is 2^-7
        check_outputs(g, r, rows=rows, o_max=2e-2, o_mean=4e-3, what=w.name)
    return g, r
