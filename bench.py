#!/usr/bin/env python
"""Throughput of tile-routed mixed-precision prefill attention on B200.

One step is one pass of the whole hot path over one batch of synthetic input already resident
in HBM: per-block 8-bit quantisation of Q and K, the routing-mask template, and the routed
attention kernel (8-bit / 16-bit QK^T tiles, shared online softmax, 16-bit P.V).  The metric is
attention TFLOP/s = 4 * D * (visible pairs) * B * H / time, reported with the realised
FP16-routed fraction and as a fraction of the blended tensor roofline
T_roof = F8 / P8 + F16 / P16 (F8: pairs of 8-bit QK tiles; F16: pairs of 16-bit QK tiles plus
all of P.V), with P16 the measured dense bf16 peak and P8 = 2 * P16 (the nominal 8-bit : 16-bit
ratio of the part).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lamp|reference]
                    [--workload long128k] [--p-fp16 P] [--tau T] [--no-sweep] [--no-extras]

The default workload is the largest single-GPU configuration, long-context prefill at
L = 131072 (B=1, H=32, Hkv=8, D=128, causal, 25% FP16 groups, swept over 0-100%).  The same
run then measures the attention kernel on the other workloads at L >= 8192 (adaptive8k with
its tau x 8-bit-format sweep, gemma_local16k, long32k, long64k) and reports them under
"other_workloads_L_ge_8192".  Each roofline fraction is given on the ruled basis (P16 = the
measured bf16 burst, P8 = 2 x P16) and, as "frac_other_bases", against the vendor library's
measured 8-bit GEMM rate (torch._int_mm / torch._scaled_mm at 8192^3) and against the rates of
the tcgen05 MMA shapes the kernel issues (the probe).

Multi-GPU (torchrun, one rank per GPU): every rank runs its own copy of the workload (independent
problems, no data-path collective: weak scaling); the timed region is bracketed by a barrier and
a device synchronise, and the slowest rank's time is used.  ``--impl reference`` times the plain
CPU oracle on sampled query rows of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_workload, sample_rows, sample_tiles  # noqa: E402

METRIC = "prefill attention TFLOP/s vs FP16-routed fraction; % of blended tensor roofline"
KERNEL_SOURCES = ["mixed_precision_tiled_b200/csrc/attn_fwd.cuh",
                  "mixed_precision_tiled_b200/csrc/attn_fwd_pp.cuh",
                  "mixed_precision_tiled_b200/csrc/ptx.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
# The headline is the largest single-GPU workload (long-context prefill at L = 131072); the
# other workloads at L >= 8192 are measured in the same run as extra keys.
DEFAULT_WORKLOAD = "long128k"
EXTRA_WORKLOADS = ["adaptive8k", "gemma_local16k", "long32k", "long64k"]


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lamp", "reference"], default="lamp")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(CONFIGS))
    ap.add_argument("--p-fp16", type=float, default=None)
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--skip-tau", type=float, default=None,
                    help="look-ahead workloads: drop tiles this far (natural log) below the "
                         "running max (threshold skip)")
    ap.add_argument("--pv8", action="store_true",
                    help="8-bit exponentials and an 8-bit P.V (E4M3 P and per-channel E4M3 V; "
                         "D = 128, the single-tile kernel); V's quantiser joins the step")
    ap.add_argument("--decode", type=int, default=0,
                    help="decode step instead of prefill: this many sequences, each with the "
                         "workload's Lk cached keys in 8 bits (INT8 KV cache), one query row per "
                         "head")
    ap.add_argument("--varlen", type=int, default=0,
                    help="run the workload's B*L query rows as a variable-length batch of this "
                         "many sequences (seeded lengths), through the packed-layout calls")
    ap.add_argument("--template", choices=["bernoulli", "sptrans"], default="bernoulli",
                    help="bitmask routing template: seeded Bernoulli groups (the workloads' "
                         "default) or the structured sink/band/stride template whose INT8 share "
                         "is 1 - FP16 fraction (--p-fp16 0.25 = SpTrans75)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other L >= 8192 workloads measured after the default one")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def describe(w, template="bernoulli", params=None) -> str:
    if w.route != "bitmask":
        route = f"adaptive tau={w.tau}"
    elif template == "sptrans":
        route = (f"bitmask g={w.group_tiles}, structured template sink/band/stride={params} "
                 f"for {1 - w.p_fp16:.0%} INT8 pairs")
    else:
        route = f"bitmask g={w.group_tiles}, {w.p_fp16:.0%} FP16 groups"
    win = f", window {w.window}" if w.window else ""
    return (f"{w.name}: B={w.B} H={w.H} Hkv={w.Hkv} Lq={w.Lq} Lk={w.Lk} D={w.D} {w.dtype}, "
            f"{'causal' if w.causal else 'non-causal'}{win}, {w.bm}x{w.bn} tiles, "
            f"{w.fmt.upper()}, {route}")


def template_params(mpt, w, p_fp16):
    """(sink, band, stride) of the structured template whose INT8 share of the visible pairs is
    closest to 1 - p_fp16 (the library's host-side search)."""
    s, b, st, _ = mpt.lamp_template_for_int8_fraction(w.Lq, w.Lk, w.D, w.group_tiles,
                                                      int(w.causal), w.window, 1.0 - p_fp16)
    return s, b, st


def tile_pairs(w) -> np.ndarray:
    """Visible (query, key) pairs of every routing tile: int64 [nQT, nKT] (geometry only)."""
    out = np.zeros((w.nqt, w.nkt), dtype=np.int64)
    c0 = np.arange(w.nkt, dtype=np.int64) * w.bn
    c1 = np.minimum(c0 + w.bn, w.Lk) - 1
    off = w.Lk - w.Lq
    for qt in range(w.nqt):
        i = np.arange(qt * w.bm, min(w.Lq, (qt + 1) * w.bm), dtype=np.int64)
        if w.causal:
            hi = np.minimum(i + off, w.Lk - 1)
            lo = np.maximum(0, i + off - w.window + 1) if w.window > 0 else np.zeros_like(i)
        else:
            hi = np.full_like(i, w.Lk - 1)
            lo = np.zeros_like(i)
        ov = np.minimum(hi[:, None], c1[None, :]) - np.maximum(lo[:, None], c0[None, :]) + 1
        out[qt] = np.clip(ov, 0, None).sum(0)
    return out


def blended_flops(w, route_map: np.ndarray, pv8: bool = False):
    """(F8, F16, F_total, 16-bit fraction): FLOPs of 8-bit QK tiles, of 16-bit QK tiles + P.V,
    the metric's FLOPs, and the fraction of visible pairs scored in 16 bits.  Route codes: 1
    8-bit, 2 16-bit by the mask, 3 recomputed by the look-ahead rule, 4 dropped by the
    threshold skip; a recomputed or dropped tile counts its 8-bit pass (the rules need the
    8-bit tile max of every tile to decide), a dropped tile has no P.V.  The metric's FLOPs
    count every visible pair.  ``pv8``: P.V runs in 8 bits and counts in F8."""
    pairs = tile_pairs(w)[None, None]  # broadcast over B, H
    p8 = int((pairs * ((route_map == 1) | (route_map == 3) | (route_map == 4))).sum())
    p16 = int((pairs * ((route_map == 2) | (route_map == 3))).sum())
    total = int((pairs * (route_map != 0)).sum())
    kept = int((pairs * ((route_map != 0) & (route_map != 4))).sum())  # P.V of kept tiles
    F8 = 2 * w.D * p8 + (2 * w.D * kept if pv8 else 0)
    F16 = 2 * w.D * p16 + (0 if pv8 else 2 * w.D * kept)
    return F8, F16, 4 * w.D * total, (p16 / total if total else 0.0)


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": m["hbm_gbs"], "bf16": m["bf16_tflops"],
                "bf16_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid, self.proc = uuid, None

    def __enter__(self):
        import threading
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        self.lines, self.t0 = [], None
        first = threading.Event()
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return self

        def reader():
            for l in self.proc.stdout:
                if l.strip():
                    self.lines.append((time.monotonic(), l))
                    first.set()
            first.set()

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        first.wait(timeout=10.0)  # sampling is running before the timed region starts
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        t1 = time.monotonic()
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        # keep the samples taken during the timed region (plus one either side)
        inside = [l for (ts, l) in self.lines if self.t0 - 0.15 <= ts <= t1 + 0.15]
        self.lines = inside or [l for (_, l) in self.lines]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def reduce_max(values, device, dist_mod=None):
    """Element-wise max of per-rank timings (the slowest rank sets the job's time)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist_mod is not None and dist_mod.is_available() and dist_mod.is_initialized() \
            and dist_mod.get_world_size() > 1:
        dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def quantiser_bandwidth(mpt, torch, dev, stream, peaks, n=20):
    """Quantiser alone on a 16-bit tensor larger than L2 (32 x 32768 x 128 bf16 = 268 MB):
    algorithmic bytes = 2 read + 1 written per element + 4 per block scale."""
    B, H, L, D = 1, 32, 32768, 128
    x = torch.randn((B, H, L, D), device=dev, dtype=torch.bfloat16)
    codes = torch.empty(x.shape, device=dev, dtype=torch.uint8)
    scales = torch.empty((B, H, L // 128), device=dev, dtype=torch.float32)
    mode = mpt.mode_bits(fmt="int8", dtype="bf16")
    for _ in range(3):
        mpt.lamp_quant_qk(x, None, codes, None, scales, None, B, H, H, L, L, D, mode, stream)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
    for i in range(n):
        ev[2 * i].record(stream)
        mpt.lamp_quant_qk(x, None, codes, None, scales, None, B, H, H, L, L, D, mode, stream)
        ev[2 * i + 1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.fmean(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n))
    nbytes = x.numel() * 3 + scales.numel() * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "quant_kernel",
            "tensor": "bf16 [1,32,32768,128] (268 MB > L2, no flush), INT8, 128-row blocks",
            "algorithmic_bytes": nbytes, "ms": round(ms, 4), "achieved_gbs": round(gbs, 1),
            "peak_gbs": peaks["hbm_gbs"], "frac": round(gbs / peaks["hbm_gbs"], 4)}


def tensor_probe(mpt, torch, stream, iters=4096):
    """Measured rate of the tcgen05 MMA shapes the attention kernel issues (one CTA per SM,
    back-to-back MMAs of M = 128 into one TMEM accumulator), in TFLOP/s (TOP/s for INT8)."""
    shapes = {"bf16_ss": (0, 16), "i8_ss": (1, 32), "bf16_ts": (2, 16)}
    nsm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    out = {}
    for name, (kind, K) in shapes.items():
        for n in (64, 128, 256):
            mpt.lamp_mma_probe(kind, n, 64, stream)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            mpt.lamp_mma_probe(kind, n, iters, stream)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            ops = 2 * 128 * n * K * 8 * iters * nsm
            out[f"{name}_n{n}"] = round(ops / (ms * 1e-3) / 1e12, 1)
    mpt.lamp_check(stream)
    return out


def attn_kernel_name(w, skip=False, pv8=False):
    """The attention kernel the library dispatches for this workload."""
    if pv8:
        return "attn_fwd_kernel (8-bit P.V)"
    wide_mask = w.route == "bitmask" and -(-w.nkt // w.group_tiles) > 128  # more than 2 words
    skip = skip and w.route == "adaptive"
    return ("attn_fwd_pp_kernel" if (w.D == 128 and w.fmt == "int8" and not wide_mask and not skip)
            else "attn_fwd_kernel")


def oracle_rows(w, n_per_head, seed):
    """Seeded query rows per (batch, head) for an oracle sample.  In adaptive mode a row's routing
    depends on every row of its query tile, so the sample is made of whole query tiles."""
    if w.route != "adaptive":
        return sample_rows(w, n_per_head, seed=seed)
    tiles = sample_tiles(w, max(1, n_per_head // w.bm), seed=seed)
    rows = (tiles[..., None] * w.bm + np.arange(w.bm)).reshape(w.B, w.H, -1)
    return np.unique(np.minimum(rows, w.Lq - 1), axis=-1) if w.Lq % w.bm else rows


def row_flops(w, rows):
    """4 * D * (visible keys) summed over the sampled rows."""
    off = w.Lk - w.Lq
    i = rows.reshape(-1).astype(np.int64)
    if not w.causal:
        return int(4 * w.D * w.Lk * i.size)
    hi = np.minimum(i + off, w.Lk - 1)
    lo = np.maximum(0, i + off - w.window + 1) if w.window > 0 else np.zeros_like(i)
    return int(4 * w.D * np.maximum(0, hi - lo + 1).sum())


def cpu_baseline(w, mask_np, t, seconds_target=15.0):
    """The oracle as it stands on a bounded sample of the workload's query rows (host cores).

    The sample grows from 4 rows per (batch, head) until one oracle call takes about
    `seconds_target` or covers every row; the last call is the one reported."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    kw = dict(bm=w.bm, bn=w.bn, causal=w.causal, window=w.window, mask=mask_np,
              group_tiles=w.group_tiles, route=w.route, fmt=w.fmt, tau=w.tau, threads=cores)
    n = 4 if w.route != "adaptive" else w.bm
    while True:
        rows = oracle_rows(w, n, seed=w.seed + 98)
        t0 = time.perf_counter()
        oracle.attention(t.q, t.k, t.v, rows=rows, **kw)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * seconds_target or rows.shape[-1] >= w.Lq:
            break
        n = min(w.Lq, max(2 * n, int(n * seconds_target / max(dt, 1e-3))))
    flops = row_flops(w, rows)
    whole = rows.shape[-1] >= w.Lq
    what = (f"the whole workload {w.name}" if whole else
            f"{rows.shape[-1]} seeded query rows per (batch, head) of {w.name}; the rate is "
            f"measured on this sample, a whole run of the workload would take "
            f"{w.flops() / (flops / dt) / 3600:.1f} h at it (extrapolated)")
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{what} ({rows.size} rows, {flops / 1e9:.1f} GFLOP, {dt:.1f} s)",
            "seconds": dt}


# ------------------------------------------------------------------ reference arm -------

def head_problem(w, t, mask, b, h):
    """The single-(batch, head) problem of query head h of batch b: the same data, B=H=Hkv=1."""
    kv = h // (w.H // w.Hkv)
    sub = w.replace(B=1, H=1, Hkv=1)
    m = mask[b:b + 1, h:h + 1] if mask is not None else None
    return sub, t.q[b:b + 1, h:h + 1], t.k[b:b + 1, kv:kv + 1], t.v[b:b + 1, kv:kv + 1], m


def run_reference(args, budget_s=90.0):
    """The oracle as it stands, timed on the host cores, on the CUDA arm's workload and metric.

    Each step runs the oracle on one seeded (batch, head) and a seeded sample of its query rows
    (whole query tiles in adaptive mode); the sample size is set during warm-up so that the whole
    run takes about `budget_s` seconds."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = CONFIGS[args.workload]
    if args.p_fp16 is not None:
        w = w.replace(p_fp16=args.p_fp16)
    if args.tau is not None:
        w = w.replace(tau=args.tau)
    t = make_workload(w)
    tp = None
    if w.route != "bitmask":
        mask = None
    elif args.template == "sptrans":
        import mixed_precision_tiled_b200 as mpt  # host-side parameter search only
        tp = template_params(mpt, w, w.p_fp16)
        mask = oracle.build_mask_template(w.B, w.H, w.Lq, w.Lk, w.bm, w.bn, w.group_tiles, *tp)
    else:
        mask = oracle.build_mask(w.B, w.H, w.nqt, w.nkt, w.group_tiles, w.p_fp16, w.mask_seed)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    per_step = max(0.01, budget_s / max(1, args.steps + args.warmup))
    n_min = w.bm if w.route == "adaptive" else 1
    n = n_min
    rng = np.random.Generator(np.random.PCG64(w.seed + 1000))
    flops_total, secs, rows_total = 0, 0.0, 0
    for s in range(args.warmup + args.steps):
        b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
        sub, q, k, v, m = head_problem(w, t, mask, b, h)
        rows = oracle_rows(sub, n, seed=w.seed + 1000 + s)
        kw = dict(bm=w.bm, bn=w.bn, causal=w.causal, window=w.window, mask=m,
                  group_tiles=w.group_tiles, route=w.route, fmt=w.fmt, tau=w.tau, threads=cores)
        t0 = time.perf_counter()
        oracle.attention(q, k, v, rows=rows, **kw)
        dt = time.perf_counter() - t0
        if s < args.warmup:  # size the per-step sample from the warm-up calls
            n = int(min(w.Lq, max(n_min, n * per_step / max(dt, 1e-4))))
            continue
        secs += dt
        rows_total += rows.size
        flops_total += row_flops(sub, rows)
    value = flops_total / secs / 1e12 if secs > 0 else 0.0
    sample = (f"per step one seeded (batch, head) of {w.name} and {n} seeded query rows of it"
              f"{' (whole query tiles)' if w.route == 'adaptive' else ''}; {args.steps} timed "
              f"steps, {rows_total} rows, {flops_total / 1e9:.2f} GFLOP, {secs:.2f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64+int64", "data": "synthetic",
            "config": {"workload": describe(w, args.template, tp)},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ CUDA arm ------------

def varlen_lengths(w, n):
    """Seeded sequence lengths (uniform in [L/4, L] before scaling) summing to B * L rows."""
    rng = np.random.Generator(np.random.PCG64(w.seed + 99))
    x = rng.uniform(0.25, 1.0, size=n)
    total = w.B * w.Lq
    lens = np.maximum(1, np.floor(x / x.sum() * total)).astype(np.int64)
    lens[-1] += total - lens.sum()
    return [int(v) for v in lens]


def run_varlen(args, w, mpt, torch, dist, dev, stream, world, rank):
    """The workload's B * L query rows as one variable-length batch (self-attention per
    sequence, causal as the workload), through lamp_quant_qk_varlen + lamp_attn_fwd_q8_varlen
    (device time) and lamp_attn_fwd_varlen with host buffers (e2e)."""
    lens = varlen_lengths(w, args.varlen)
    B, H, Hkv, D = len(lens), w.H, w.Hkv, w.D
    L = max(lens)
    total = sum(lens)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    q = torch.randn((H, total, D), generator=gen).to(tdt).to(dev)
    k = torch.randn((Hkv, total, D), generator=gen).to(tdt).to(dev)
    v = torch.randn((Hkv, total, D), generator=gen).to(tdt).to(dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    bm, bn = w.bm, w.bn
    nqt, nkt = -(-L // bm), -(-L // bn)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
    qs = torch.empty((B, H, nqt), dtype=torch.float32, device=dev)
    ks = torch.empty((B, Hkv, nkt), dtype=torch.float32, device=dev)
    bitmask = w.route == "bitmask"
    W = mpt.lamp_mask_words(L, D, w.group_tiles)
    mask = torch.empty((B, H, nqt, W), dtype=torch.int64, device=dev)
    o = torch.empty((H, total, D), dtype=torch.float32, device=dev)
    lse = torch.empty((H, total), dtype=torch.float32, device=dev)
    mode = mpt.mode_bits(w.route, w.fmt, w.dtype)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(ev_a=None, ev_b=None):
        mpt.lamp_quant_qk_varlen(q, k, q8, k8, qs, ks, cu, cu, B, H, Hkv, L, L, total, total, D,
                                 mode, stream)
        if bitmask:
            mpt.lamp_build_mask(mask, B, H, L, L, D, w.group_tiles, w.p_fp16, w.mask_seed, stream)
        if ev_a is not None:
            ev_a.record(stream)
        mpt.lamp_attn_fwd_q8_varlen(q, k, v, q8, k8, qs, ks, o, lse, cu, cu, B, H, Hkv, L, L,
                                    total, total, D, int(w.causal), w.window, 0.0,
                                    mask if bitmask else None, w.group_tiles, mode, w.tau, None,
                                    stream)
        if ev_b is not None:
            ev_b.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    mpt.lamp_check(stream)
    rmap = torch.empty((B, H, nqt, nkt), dtype=torch.uint8, device=dev)
    mpt.lamp_attn_fwd_q8_varlen(q, k, v, q8, k8, qs, ks, o, lse, cu, cu, B, H, Hkv, L, L, total,
                                total, D, int(w.causal), w.window, 0.0, mask if bitmask else None,
                                w.group_tiles, mode, w.tau, rmap, stream)
    torch.cuda.synchronize()
    rm = rmap.cpu().numpy()
    F8 = F16 = F = 0
    for b, n in enumerate(lens):
        wb = w.replace(B=1, Lq=n, Lk=n)
        f8, f16, f, _ = blended_flops(wb, rm[b:b + 1, :, :wb.nqt, :wb.nkt])
        F8, F16, F = F8 + f8, F16 + f16, F + f
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    if world > 1:
        dist.barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(uuid if rank == 0 else None) as clk:
        for i in range(args.steps):
            flush.zero_()
            flush.view(torch.int64).sum()
            ev[i][0].record(stream)
            step(ev[i][1], ev[i][2])
            ev[i][3].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    mpt.lamp_check(stream)
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    tot_ms, att_ms = reduce_max([sum(step_ms), statistics.fmean(attn_ms)], dev, dist)
    ms_per_step = tot_ms / args.steps
    # end to end: pinned host buffers in, O and lse out
    hq = torch.empty(q.shape, dtype=tdt, pin_memory=True).copy_(q)
    hk = torch.empty(k.shape, dtype=tdt, pin_memory=True).copy_(k)
    hv = torch.empty(v.shape, dtype=tdt, pin_memory=True).copy_(v)
    ho = torch.empty(o.shape, dtype=torch.float32, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        if bitmask:
            mpt.lamp_build_mask(mask, B, H, L, L, D, w.group_tiles, w.p_fp16, w.mask_seed, stream)
        mpt.lamp_attn_fwd_varlen(dq, dk, dv, o, lse, cu, cu, B, H, Hkv, L, L, total, total, D,
                                 int(w.causal), w.window, 0.0, mask if bitmask else None,
                                 w.group_tiles, mode, w.tau, stream)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = reduce_max([e0.elapsed_time(e1) / n_e2e], dev, dist)
    peaks = measured_peaks()
    P16 = peaks["bf16"] * 1e12
    T_roof = F8 / (2.0 * P16) + F16 / P16
    achieved = F / (att_ms * 1e-3) / 1e12
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(world * F / (ms_per_step * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": f"int8+{w.dtype}" if w.fmt == "int8" else f"e4m3+{w.dtype}",
            "data": "synthetic",
            "config": {"workload": describe(w) + f"; as a variable-length batch of {B} sequences",
                       "lengths": lens, "fp16_fraction_realised": round(2.0 * F16 / F - 1.0, 4) if F else 0.0,
                       "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed between steps (256 MiB write, then read back); per-step CUDA events exclude the flush"},
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                         "peak": round(F / T_roof / 1e12, 1), "unit": "TFLOP/s",
                         "frac": round(T_roof / (att_ms * 1e-3), 4), "traffic": None,
                         "peak_basis": f"blended: F8/P8 + F16/P16, P16 = {peaks['bf16']} TFLOP/s "
                                       f"bf16 burst ({peaks['source']}), P8 = 2 x P16 (nominal ratio)",
                         "kernel": attn_kernel_name(w), "attn_ms": round(att_ms, 4)},
            "e2e": {"value": round(F * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * q.element_size(),
                    "d2h_bytes_per_step": o.numel() * 4 + lse.numel() * 4,
                    "ms_per_step": round(e2e_ms, 4)},
            "clocks": clk.summary(),
            "gpu_launches": (3 if bitmask else 2) * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_decode(args, w, mpt, torch, dist, dev, stream, world, rank):
    """One decode step: args.decode sequences with w.Lk cached keys each (8-bit K and V with
    per-block scales, the workload's format), one query row per head, bitmask routing with the
    workload's group size and FP16 fraction.  The kernel reads the cache once: bound by HBM."""
    B, H, Hkv, D, L = args.decode, w.H, w.Hkv, w.D, w.Lk
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    q = torch.randn((B, H, 1, D), generator=gen).to(tdt).to(dev)
    kv = torch.randn((B, Hkv, L, D), generator=gen).to(tdt).to(dev)
    nkt = -(-L // w.bn)
    mode = mpt.mode_bits("bitmask", w.fmt, w.dtype)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    qs = torch.empty((B, H, 1), dtype=torch.float32, device=dev)
    k8 = torch.empty(kv.shape, dtype=torch.uint8, device=dev)
    v8 = torch.empty(kv.shape, dtype=torch.uint8, device=dev)
    ks = torch.empty((B, Hkv, nkt), dtype=torch.float32, device=dev)
    vs = torch.empty((B, Hkv, nkt), dtype=torch.float32, device=dev)
    mpt.lamp_quant_qk(None, kv, None, k8, None, ks, B, H, Hkv, 1, L, D, mode, stream)
    kv.copy_(torch.randn(kv.shape, generator=gen).to(tdt))
    mpt.lamp_quant_qk(None, kv, None, v8, None, vs, B, H, Hkv, 1, L, D, mode, stream)
    del kv
    W = mpt.lamp_mask_words(L, D, w.group_tiles)
    mask = torch.empty((B, H, 1, W), dtype=torch.int64, device=dev)
    mpt.lamp_build_mask(mask, B, H, 1, L, D, w.group_tiles, w.p_fp16, w.mask_seed, stream)
    o = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(ev_a=None, ev_b=None):
        mpt.lamp_quant_qk(q, None, q8, None, qs, None, B, H, Hkv, 1, L, D, mode, stream)
        if ev_a is not None:
            ev_a.record(stream)
        mpt.lamp_decode_fwd(q, q8, qs, k8, ks, v8, vs, None, o, lse, B, H, Hkv, L, D, 0.0, mask,
                            w.group_tiles, mode, stream)
        if ev_b is not None:
            ev_b.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    mpt.lamp_check(stream)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    if world > 1:
        dist.barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(uuid if rank == 0 else None) as clk:
        for i in range(args.steps):
            flush.zero_()
            flush.view(torch.int64).sum()
            ev[i][0].record(stream)
            step(ev[i][1], ev[i][2])
            ev[i][3].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    mpt.lamp_check(stream)
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    tot_ms, d_ms = reduce_max([sum(step_ms), statistics.fmean(dec_ms)], dev, dist)
    ms_per_step = tot_ms / args.steps
    F = 4 * D * H * B * L  # one query row per head over L keys
    cache_bytes = 2 * B * Hkv * L * D + 2 * B * Hkv * nkt * 4
    peaks = measured_peaks()
    gbs = cache_bytes / (d_ms * 1e-3) / 1e9
    # end to end: the query in from pinned host memory, O and lse out
    hq = torch.empty(q.shape, dtype=tdt, pin_memory=True).copy_(q)
    ho = torch.empty(o.shape, dtype=torch.float32, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = reduce_max([e0.elapsed_time(e1) / n_e2e], dev, dist)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(world * F / (ms_per_step * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": f"int8+{w.dtype}" if w.fmt == "int8" else f"e4m3+{w.dtype}",
            "data": "synthetic",
            "config": {"workload": f"decode: {B} sequences x {L} cached keys (8-bit K and V), "
                                   f"H={H} Hkv={Hkv} D={D}, one query row per head, "
                                   f"bitmask g={w.group_tiles}, {w.p_fp16:.0%} FP16 groups",
                       "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed between steps (256 MiB write, then read back); per-step CUDA events exclude the flush"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None,
                         "algorithmic_bytes": cache_bytes,
                         "peak_basis": f"copy bandwidth ({peaks['source']})",
                         "kernel": "decode_split_kernel + decode_combine_kernel",
                         "decode_ms": round(d_ms, 4)},
            "e2e": {"value": round(F * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": q.numel() * q.element_size(),
                    "d2h_bytes_per_step": o.numel() * 4 + lse.numel() * 4,
                    "ms_per_step": round(e2e_ms, 4)},
            "clocks": clk.summary(),
            "gpu_launches": 3 * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def library_peaks(torch, dev, n=8192, reps=10):
    """Dense 8-bit GEMM rates of the vendor library at n^3 (best of `reps`, CUDA events): INT8
    by torch._int_mm, FP8 E4M3 by torch._scaled_mm (bf16 output, unit scales), and bf16 by
    torch.matmul, in TOP/s / TFLOP/s (2 n^3 operations).  These are denominators only."""
    out = {}
    g = torch.Generator(device=dev).manual_seed(0)

    def best(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return round(2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12, 1)

    try:
        a = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g)
        b = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g)
        out["int8_int_mm"] = best(lambda: torch._int_mm(a, b))
        del a, b
    except Exception as e:  # noqa: BLE001  (report, do not fail the bench)
        out["int8_int_mm_error"] = str(e)[:200]
    try:
        a = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        out["e4m3_scaled_mm"] = best(lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,
                                                               out_dtype=torch.bfloat16))
        del a, b
    except Exception as e:  # noqa: BLE001
        out["e4m3_scaled_mm_error"] = str(e)[:200]
    a = torch.randn((n, n), device=dev, generator=g, dtype=torch.bfloat16)
    b = torch.randn((n, n), device=dev, generator=g, dtype=torch.bfloat16)
    out["bf16_matmul"] = best(lambda: torch.matmul(a, b))
    del a, b
    torch.cuda.empty_cache()
    return out


def roofline_fracs(F8, F16, attn_ms, peaks, fmt, lib=None, probe=None):
    """Blended-roofline fractions of one attention launch: T_roof / measured time, with
    T_roof = F8 / P8 + F16 / P16 on three bases: the ruled one (P16 = the measured bf16 burst,
    P8 = 2 x P16), the vendor library's measured 8-bit GEMM rate for P8 (bf16 unchanged), and
    the tcgen05 probe's rates for both (the MMA shapes the kernel issues)."""
    t = attn_ms * 1e-3
    P16 = peaks["bf16"] * 1e12
    out = {"ruled": (F8 / (2.0 * P16) + F16 / P16) / t}
    key = "int8_int_mm" if fmt == "int8" else "e4m3_scaled_mm"
    if lib and key in lib:
        out["library_8bit"] = (F8 / (lib[key] * 1e12) + F16 / P16) / t
    if probe and "i8_ss_n128" in probe and "bf16_ss_n128" in probe:
        # (no E4M3 probe kind: kind::f8f6f4 and kind::i8 have the same dense rate on this part)
        out["tcgen05_probe"] = (F8 / (probe["i8_ss_n128"] * 1e12)
                                + F16 / (probe["bf16_ss_n128"] * 1e12)) / t
    return {k: round(v, 4) for k, v in out.items()}


def traffic_record(w):
    try:
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        rec = tr.get("records", {}).get(w.name)
        if rec and tr.get("kernel_hash") == kernel_hash():
            return rec.get("traffic_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


class Prefill:
    """One workload on the device: inputs resident in HBM, the step (quantiser, routing mask,
    attention kernel), its timing and the route map behind the blended roofline."""

    def __init__(self, args, w, mpt, torch, dev, stream, t=None):
        self.args, self.w, self.mpt, self.torch, self.dev, self.stream = args, w, mpt, torch, dev, stream
        self.t = make_workload(w) if t is None else t
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
        self.tdt = tdt

        def dev16(bits):
            return torch.from_numpy(bits.view(np.int16)).view(tdt).to(dev)

        self.q, self.k, self.v = dev16(self.t.q_bits), dev16(self.t.k_bits), dev16(self.t.v_bits)
        B, H, Hkv = w.B, w.H, w.Hkv
        self.mode = mpt.mode_bits(w.route, w.fmt, w.dtype)
        self.q8 = torch.empty(self.q.shape, dtype=torch.uint8, device=dev)
        self.k8 = torch.empty(self.k.shape, dtype=torch.uint8, device=dev)
        self.qs = torch.empty((B, H, w.nqt), dtype=torch.float32, device=dev)
        self.ks = torch.empty((B, Hkv, w.nkt), dtype=torch.float32, device=dev)
        W = mpt.lamp_mask_words(w.Lk, w.D, w.group_tiles)
        self.mask = torch.empty((B, H, w.nqt, W), dtype=torch.int64, device=dev)
        self.o = torch.empty((B, H, w.Lq, w.D), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B, H, w.Lq), dtype=torch.float32, device=dev)
        self.rmap = torch.empty((B, H, w.nqt, w.nkt), dtype=torch.uint8, device=dev)
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 256 MiB > 126 MB L2
        self.bitmask = w.route == "bitmask"
        self.skip = args.skip_tau is not None and not self.bitmask
        self.tparams = {}
        self.launches_per_step = 1 + (1 if self.bitmask else 0) + 1  # quantiser, mask, attention
        self.pv8 = bool(getattr(args, "pv8", False))
        if self.pv8:  # V's quantiser (three kernels) joins the step
            self.mode |= mpt.PV_E4M3
            self.v8t = torch.empty((B, Hkv, w.D, (w.Lk + 15) // 16 * 16), dtype=torch.uint8,
                                   device=dev)
            self.vs = torch.empty((B, Hkv, w.D), dtype=torch.float32, device=dev)
            self.launches_per_step += 3

    def flush_l2(self):
        """Evict the previous step's lines: write 256 MiB, then read it back so that L2 holds
        clean lines only (no write-back of the flush lands in the next timed step)."""
        self.flush.zero_()
        self.flush.view(self.torch.int64).sum()

    def build_mask(self, pf):
        w, mpt = self.w, self.mpt
        if self.args.template == "sptrans":
            if pf not in self.tparams:
                self.tparams[pf] = template_params(mpt, w, pf)
            mpt.lamp_build_mask_template(self.mask, w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles,
                                         *self.tparams[pf], self.stream)
        else:
            mpt.lamp_build_mask(self.mask, w.B, w.H, w.Lq, w.Lk, w.D, w.group_tiles, pf,
                                w.mask_seed, self.stream)

    def attn(self, md, tu, route_out=None):
        w, mpt = self.w, self.mpt
        if self.pv8 and route_out is None:
            mpt.lamp_attn_fwd_q8_pv8(self.q, self.k, self.q8, self.k8, self.qs, self.ks, self.v8t,
                                     self.vs, self.o, self.lse, w.B, w.H, w.Hkv, w.Lq, w.Lk, w.D,
                                     int(w.causal), w.window, 0.0,
                                     self.mask if self.bitmask else None, w.group_tiles,
                                     md | mpt.PV_E4M3, tu, self.stream)
            return
        md &= ~mpt.PV_E4M3  # the route map comes from the 16-bit P kernel: the same decisions
        if self.skip:
            mpt.lamp_attn_fwd_q8_skip(self.q, self.k, self.v, self.q8, self.k8, self.qs, self.ks,
                                      self.o, self.lse, w.B, w.H, w.Hkv, w.Lq, w.Lk, w.D,
                                      int(w.causal), w.window, 0.0, md, tu, self.args.skip_tau,
                                      route_out, self.stream)
        else:
            mpt.lamp_attn_fwd_q8(self.q, self.k, self.v, self.q8, self.k8, self.qs, self.ks,
                                 self.o, self.lse, w.B, w.H, w.Hkv, w.Lq, w.Lk, w.D,
                                 int(w.causal), w.window, 0.0,
                                 self.mask if self.bitmask else None, w.group_tiles, md, tu,
                                 route_out, self.stream)

    def step(self, ev_a=None, ev_b=None, p_fp16=None, mode_=None, tau_=None):
        w = self.w
        md = self.mode if mode_ is None else mode_
        tu = w.tau if tau_ is None else tau_
        self.mpt.lamp_quant_qk(self.q, self.k, self.q8, self.k8, self.qs, self.ks, w.B, w.H,
                               w.Hkv, w.Lq, w.Lk, w.D, md, self.stream)
        if self.pv8:
            self.mpt.lamp_quant_v(self.v, self.v8t, self.vs, w.B, w.Hkv, w.Lk, w.D, md, self.stream)
        if self.bitmask:
            self.build_mask(w.p_fp16 if p_fp16 is None else p_fp16)
        if ev_a is not None:
            ev_a.record(self.stream)
        self.attn(md, tu)
        if ev_b is not None:
            ev_b.record(self.stream)

    def timed(self, n, **kw):
        """Per-step and attention-kernel device times (ms) over n steps, L2 flushed between."""
        torch = self.torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for i in range(n):
            self.flush_l2()
            ev[i][0].record(self.stream)
            self.step(ev[i][1], ev[i][2], **kw)
            ev[i][3].record(self.stream)
        torch.cuda.synchronize()
        return ([ev[i][0].elapsed_time(ev[i][3]) for i in range(n)],
                [ev[i][1].elapsed_time(ev[i][2]) for i in range(n)])

    def route_flops(self, p_fp16=None, mode_=None, tau_=None):
        """(F8, F16, F, 16-bit fraction, route map) of the configuration (one untimed call)."""
        w = self.w
        self.step(p_fp16=p_fp16, mode_=mode_, tau_=tau_)
        self.attn(self.mode if mode_ is None else mode_, w.tau if tau_ is None else tau_,
                  self.rmap)
        self.torch.cuda.synchronize()
        rm = self.rmap.cpu().numpy()
        return (*blended_flops(w, rm, self.pv8), rm)

    def sweep(self, peaks, lib, probe):
        """FP16-fraction sweep (bitmask) or tau x 8-bit-format sweep with the rerouted fraction
        (look-ahead), each point timed on its own."""
        w, mpt, out = self.w, self.mpt, {}
        n = 10 if w.flops() > 5e12 else max(20, self.args.steps // 10)
        if self.bitmask:
            for pf in (0.0, 0.1, 0.25, 0.5, 1.0):
                f8, f16, ff, fr, _ = self.route_flops(p_fp16=pf)
                _, at = self.timed(n, p_fp16=pf)
                a = float(statistics.fmean(at))
                out[f"{pf:g}"] = {"fp16_fraction_realised": round(fr, 4),
                                  "attn_tflops": round(ff / (a * 1e-3) / 1e12, 1),
                                  "roofline_frac": roofline_fracs(f8, f16, a, peaks, w.fmt, lib,
                                                                  probe)["ruled"]}
        else:
            for fmt in ("int8", "e4m3"):
                md = mpt.mode_bits(w.route, fmt, w.dtype, pv8=self.pv8)
                for tau in (0.5, 1.0, 2.0, 4.0, 8.0):
                    f8, f16, ff, fr, _ = self.route_flops(mode_=md, tau_=tau)
                    _, at = self.timed(n, mode_=md, tau_=tau)
                    a = float(statistics.fmean(at))
                    out[f"{fmt} tau={tau:g}"] = {
                        "rerouted_fraction": round(fr, 4),
                        "attn_tflops": round(ff / (a * 1e-3) / 1e12, 1),
                        "roofline_frac": roofline_fracs(f8, f16, a, peaks, fmt, lib, probe)["ruled"],
                        "kernel": attn_kernel_name(w.replace(fmt=fmt), pv8=self.pv8)}
        self.step()  # restore the configured mask / format / tau
        self.torch.cuda.synchronize()
        return out

    def release(self):
        for name in ("q", "k", "v", "q8", "k8", "qs", "ks", "mask", "o", "lse", "rmap", "flush",
                     "v8t", "vs"):
            setattr(self, name, None)
        self.torch.cuda.empty_cache()


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import mixed_precision_tiled_b200 as mpt

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    w = CONFIGS[args.workload]
    if args.p_fp16 is not None:
        w = w.replace(p_fp16=args.p_fp16)
    if args.tau is not None:
        w = w.replace(tau=args.tau)
    if args.varlen > 0:
        return run_varlen(args, w, mpt, torch, dist, dev, stream, world, rank)
    if args.decode > 0:
        return run_decode(args, w, mpt, torch, dist, dev, stream, world, rank)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    peaks = measured_peaks()
    P = Prefill(args, w, mpt, torch, dev, stream)
    B, H, Hkv, Lq, Lk, D = w.B, w.H, w.Hkv, w.Lq, w.Lk, w.D

    for _ in range(args.warmup):
        P.step()
    torch.cuda.synchronize()
    mpt.lamp_check(stream)
    F8, F16, F, frac16, rm = P.route_flops()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid if rank == 0 else None) as clk:
        step_ms, attn_ms = P.timed(args.steps)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    mpt.lamp_check(stream)
    tot_ms, att_ms = reduce_max([sum(step_ms), statistics.fmean(attn_ms)], dev, dist)
    ms_per_step = tot_ms / args.steps
    value = world * F / (ms_per_step * 1e-3) / 1e12

    # end-to-end through the public C-ABI call on pinned host buffers: lamp_attn_fwd_host copies
    # Q, K, V in, quantises, attends and copies O and lse out, chunk by chunk, the copies of one
    # chunk overlapping the compute of the next
    tdt = P.tdt
    hq = torch.empty(P.q.shape, dtype=tdt, pin_memory=True).copy_(P.q)
    hk = torch.empty(P.k.shape, dtype=tdt, pin_memory=True).copy_(P.k)
    hv = torch.empty(P.v.shape, dtype=tdt, pin_memory=True).copy_(P.v)
    ho = torch.empty(P.o.shape, dtype=torch.float32, pin_memory=True)
    hl = torch.empty(P.lse.shape, dtype=torch.float32, pin_memory=True)

    def e2e_step():
        if P.bitmask:
            P.build_mask(w.p_fp16)
        mpt.lamp_attn_fwd_host(hq, hk, hv, ho, hl, B, H, Hkv, Lq, Lk, D, int(w.causal), w.window,
                               0.0, P.mask if P.bitmask else None, w.group_tiles, P.mode, w.tau,
                               0, stream)

    n_e2e = max(3, min(args.steps, 30))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = reduce_max([e0.elapsed_time(e1) / n_e2e], dev, dist)
    mpt.lamp_check(stream)
    h2d = (P.q.numel() + P.k.numel() + P.v.numel()) * P.q.element_size()
    d2h = P.o.numel() * 4 + P.lse.numel() * 4
    del hq, hk, hv, ho, hl

    lib = library_peaks(torch, dev) if not args.no_sweep else None
    probe = tensor_probe(mpt, torch, stream) if not args.no_sweep else None
    sweep = P.sweep(peaks, lib, probe) if not args.no_sweep else {}
    quant = quantiser_bandwidth(mpt, torch, dev, stream, peaks) if not args.no_sweep else None

    fr = roofline_fracs(F8, F16, att_ms, peaks, w.fmt, lib, probe)
    achieved = F / (att_ms * 1e-3) / 1e12
    T_roof = F8 / (2.0 * peaks["bf16"] * 1e12) + F16 / (peaks["bf16"] * 1e12)
    mask_np = P.mask.cpu().numpy().view(np.uint64) if P.bitmask else None
    dropped = round(float((tile_pairs(w)[None, None] * (rm == 4)).sum()) / max(1, F // (4 * w.D)), 4)
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"int8+{w.dtype}" if w.fmt == "int8" else f"e4m3+{w.dtype}",
        "data": "synthetic",
        "config": {"workload": describe(w, args.template, P.tparams.get(w.p_fp16))
                               + (f", threshold skip {args.skip_tau}" if P.skip else ""),
                   "fp16_fraction_realised": round(frac16, 4),
                   "dropped_fraction": dropped,
                   "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed between steps (256 MiB write, then read back); per-step CUDA "
                         "events exclude the flush"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": round(F / T_roof / 1e12, 1), "unit": "TFLOP/s",
                     "frac": fr["ruled"], "traffic": None if P.pv8 else traffic_record(w),
                     "peak_basis": f"blended: F8/P8 + F16/P16, P16 = {peaks['bf16']} TFLOP/s bf16 "
                                   f"burst ({peaks['source']}), P8 = 2 x P16 (nominal ratio)"
                                   + ("; P.V counted in F8" if P.pv8 else ""),
                     "frac_other_bases": {k: v for k, v in fr.items() if k != "ruled"},
                     "kernel": attn_kernel_name(w, args.skip_tau is not None, P.pv8),
                     "attn_ms": round(att_ms, 4)},
        "e2e": {"value": round(F * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "clocks": clocks,
        "gpu_launches": P.launches_per_step * args.steps,
    }
    if clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        # the same fraction against the peaks scaled to the SM clock seen under load (a kernel
        # running under the power cap cannot reach the burst-clock peak)
        line["roofline"]["frac_at_observed_clock"] = round(
            fr["ruled"] * clocks["sm_max_mhz"] / clocks["sm_mhz"], 4)
    if sweep:
        line["sweep_fp16_fraction" if P.bitmask else "sweep_tau_format"] = sweep
    if quant:
        line["quantiser"] = quant
    if probe:
        line["tensor_probe_tflops"] = probe
    if lib:
        line["library_gemm_tflops"] = lib
    t_host = P.t
    P.release()

    # the other workloads at L >= 8192 (the target's configurations), kernel-level, same run
    if (not args.no_extras and args.workload == DEFAULT_WORKLOAD and args.varlen == 0
            and not args.pv8):
        extras = {}
        for name in EXTRA_WORKLOADS:
            we = CONFIGS[name]
            X = Prefill(args, we, mpt, torch, dev, stream)
            for _ in range(max(3, min(args.warmup, 5))):
                X.step()
            torch.cuda.synchronize()
            f8, f16, ff, fr16, rme = X.route_flops()
            n = max(3, min(args.steps, 20))
            with ClockSampler(uuid if rank == 0 else None) as clk_e:
                st_ms, at_ms = X.timed(n)
            mpt.lamp_check(stream)
            a = float(statistics.fmean(at_ms))
            s_ms = float(statistics.fmean(st_ms))
            fre = roofline_fracs(f8, f16, a, peaks, we.fmt, lib, probe)
            ex = {"workload": describe(we), "steps": n,
                  "step_tflops": round(ff / (s_ms * 1e-3) / 1e12, 1),
                  "attn_tflops": round(ff / (a * 1e-3) / 1e12, 1), "attn_ms": round(a, 4),
                  ("fp16_fraction_realised" if we.route == "bitmask" else "rerouted_fraction"):
                      round(fr16, 4),
                  "roofline_frac": fre["ruled"],
                  "frac_other_bases": {k: v for k, v in fre.items() if k != "ruled"},
                  "kernel": attn_kernel_name(we), "traffic": traffic_record(we),
                  "clocks": clk_e.summary()}
            if not args.no_sweep:
                ex["sweep_fp16_fraction" if X.bitmask else "sweep_tau_format"] = X.sweep(peaks, lib, probe)
            extras[name] = ex
            X.release()
            del X
        line["other_workloads_L_ge_8192"] = extras

    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            import oracle  # noqa: F401  (CPU baseline leg only)
            line["cpu_baseline"] = cpu_baseline(w, mask_np, t_host)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
