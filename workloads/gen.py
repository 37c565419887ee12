"""Seeded synthetic inputs shaped like the pages' prefill workloads.

The pages measure on real models (TileMix: LLaMA/Qwen/Vicuna prefill at 4k/8k and LV-Eval
long-context inputs; LampAttention: Qwen3 and Gemma 3).  No weights or datasets are used here:
these generators stand in for them with the same shapes and with the structure that makes
tile routing matter -- per-channel scale spread, a few outlier channels per head, planted
"retrieval" keys that one query row attends to sharply, and an attention-sink key.

Recipe (every draw comes from one numpy PCG64 stream seeded per workload):
  * V is i.i.d. N(0, 1) everywhere.
  * "iid" workloads: Q, K i.i.d. N(0, 1).
  * "structured" workloads: Q = N(0,1) * sigma[h, c] with sigma log-normal(0, 0.5) drawn per
    (Q head, channel); K the same with its own sigma per (KV head, channel); 4 distinct
    outlier channels per head (drawn independently for Q and K) get sigma * 20.
  * planted retrievals: for a fraction of query rows, drawn per (batch, KV head) without
    replacement, one key j that the row can see (causal / window visibility, j != i) is set to
    4 * unit(q_i), q_i taken from the first Q head of the group.  Later plants overwrite
    earlier ones.
  * sink: key 0 of every KV head scaled by 6.
  * all values are drawn in fp32 and rounded to nearest-even into fp16 or bf16; the returned
    fp32 arrays hold exactly the 16-bit values.

Nothing in this module quantises, routes, scores or normalises: it only produces inputs.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    Lq: int
    Lk: int
    D: int
    bm: int
    bn: int
    causal: bool
    window: int
    dtype: str            # "fp16" | "bf16"
    route: str            # "bitmask" | "adaptive"
    fmt: str              # "int8" | "e4m3"
    group_tiles: int
    p_fp16: float
    tau: float
    seed: int
    values: str           # "iid" | "structured"
    plant_frac: float = 0.0
    sink: bool = False

    @property
    def mask_seed(self) -> int:
        return self.seed + 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # ---- geometry (pure bookkeeping, no method arithmetic) ----
    @property
    def nqt(self) -> int:
        return -(-self.Lq // self.bm)

    @property
    def nkt(self) -> int:
        return -(-self.Lk // self.bn)

    def visible(self, i: int):
        """Inclusive key range [lo, hi] that query row i may see (empty if lo > hi)."""
        if not self.causal:
            return 0, self.Lk - 1
        hi = min(i + (self.Lk - self.Lq), self.Lk - 1)
        lo = 0 if self.window <= 0 else max(0, i + (self.Lk - self.Lq) - self.window + 1)
        return lo, hi

    def pairs(self) -> int:
        """Number of visible (query, key) pairs per (batch, head)."""
        if not self.causal:
            return self.Lq * self.Lk
        off = self.Lk - self.Lq
        tot = 0
        # closed form per row is cheap enough even at 131072 rows with numpy
        i = np.arange(self.Lq, dtype=np.int64)
        hi = np.minimum(i + off, self.Lk - 1)
        lo = np.zeros_like(i) if self.window <= 0 else np.maximum(0, i + off - self.window + 1)
        tot = int(np.clip(hi - lo + 1, 0, None).sum())
        return tot

    def flops(self) -> int:
        """4 * D * pairs * B * H (QK^T and P.V, causal/window-adjusted)."""
        return 4 * self.D * self.pairs() * self.B * self.H


def _cfg(**kw) -> Workload:
    return Workload(**kw)


# The five workloads of the build's scope table.  Config texts call the GQA workload
# "config 1"; the tiny check is config 0.
CONFIGS = {
    "tiny": _cfg(name="tiny", B=1, H=1, Hkv=1, Lq=256, Lk=256, D=64, bm=64, bn=64,
                 causal=False, window=0, dtype="fp16", route="bitmask", fmt="int8",
                 group_tiles=1, p_fp16=0.25, tau=0.0, seed=1000, values="iid"),
    "gqa4k": _cfg(name="gqa4k", B=1, H=32, Hkv=8, Lq=4096, Lk=4096, D=128, bm=128, bn=128,
                  causal=True, window=0, dtype="bf16", route="bitmask", fmt="int8",
                  group_tiles=4, p_fp16=0.20, tau=0.0, seed=1001, values="structured",
                  plant_frac=0.01),
    "adaptive8k": _cfg(name="adaptive8k", B=2, H=32, Hkv=8, Lq=8192, Lk=8192, D=128,
                       bm=128, bn=128, causal=True, window=0, dtype="bf16", route="adaptive",
                       fmt="e4m3", group_tiles=1, p_fp16=0.0, tau=4.0, seed=1002,
                       values="structured", plant_frac=0.02),
    "gemma_local16k": _cfg(name="gemma_local16k", B=1, H=8, Hkv=4, Lq=16384, Lk=16384, D=256,
                           bm=64, bn=128, causal=True, window=1024, dtype="bf16",
                           route="bitmask", fmt="int8", group_tiles=2, p_fp16=0.30, tau=0.0,
                           seed=1003, values="structured", plant_frac=0.01, sink=True),
    "long32k": _cfg(name="long32k", B=1, H=32, Hkv=8, Lq=32768, Lk=32768, D=128, bm=128,
                    bn=128, causal=True, window=0, dtype="bf16", route="bitmask", fmt="int8",
                    group_tiles=8, p_fp16=0.25, tau=0.0, seed=1004, values="structured",
                    plant_frac=0.001),
}
CONFIGS["long64k"] = CONFIGS["long32k"].replace(name="long64k", Lq=65536, Lk=65536)
CONFIGS["long128k"] = CONFIGS["long32k"].replace(name="long128k", Lq=131072, Lk=131072)


def config_by_name(name: str) -> Workload:
    return CONFIGS[name]


def _chunked(fn, n: int, chunk: int = 1 << 24):
    """Runs fn(lo, hi) over [0, n) in chunks on a thread pool (numpy's element-wise kernels
    release the GIL); the result does not depend on the chunking."""
    if n <= chunk:
        fn(0, n)
        return
    from concurrent.futures import ThreadPoolExecutor
    import os
    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda lo: fn(lo, min(n, lo + chunk)), range(0, n, chunk)))


def _round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).reshape(-1)
    out = np.empty(u.shape, dtype=np.uint16)

    def part(lo, hi):
        v = u[lo:hi]
        r = ((v >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
        out[lo:hi] = (v + r) >> np.uint32(16)

    _chunked(part, u.size)
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    flat = np.ascontiguousarray(b).reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint32)

    def part(lo, hi):
        out[lo:hi] = flat[lo:hi].astype(np.uint32) << np.uint32(16)

    _chunked(part, flat.size)
    return out.view(np.float32).reshape(b.shape)


def to_16bit(x: np.ndarray, dtype: str):
    """Round fp32 to the 16-bit input type.  Returns (bits uint16, exact fp32 values)."""
    if dtype == "fp16":
        h = x.astype(np.float16)
        return h.view(np.uint16), h.astype(np.float32)
    if dtype == "bf16":
        b = _round_bf16(x)
        return b, bf16_bits_to_f32(b)
    raise ValueError(dtype)


@dataclasses.dataclass
class Tensors:
    """Inputs of one workload: 16-bit bit patterns (for the GPU) and their exact fp32 values."""
    q_bits: np.ndarray
    k_bits: np.ndarray
    v_bits: np.ndarray
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray


def make_workload(w: Workload, *, v_ones: bool = False) -> Tensors:
    rng = np.random.Generator(np.random.PCG64(w.seed))
    G = w.H // w.Hkv
    q = rng.standard_normal((w.B, w.H, w.Lq, w.D), dtype=np.float32)
    k = rng.standard_normal((w.B, w.Hkv, w.Lk, w.D), dtype=np.float32)
    v = rng.standard_normal((w.B, w.Hkv, w.Lk, w.D), dtype=np.float32)
    if w.values == "structured":
        sig_q = np.exp(0.5 * rng.standard_normal((w.H, w.D))).astype(np.float32)
        sig_k = np.exp(0.5 * rng.standard_normal((w.Hkv, w.D))).astype(np.float32)
        for h in range(w.H):
            sig_q[h, rng.choice(w.D, size=4, replace=False)] *= 20.0
        for h in range(w.Hkv):
            sig_k[h, rng.choice(w.D, size=4, replace=False)] *= 20.0
        q *= sig_q[None, :, None, :]
        k *= sig_k[None, :, None, :]
        if w.plant_frac > 0:
            n_plant = int(round(w.plant_frac * w.Lq))
            for b in range(w.B):
                for kh in range(w.Hkv):
                    rows = rng.choice(w.Lq, size=n_plant, replace=False)
                    u = rng.random(n_plant)
                    for i, ui in zip(rows.tolist(), u.tolist()):
                        lo, hi = w.visible(i)
                        cand = hi - lo + 1 - (1 if lo <= i <= hi else 0)
                        if cand <= 0:
                            continue
                        t = min(int(ui * cand), cand - 1)
                        j = lo + t
                        if lo <= i <= hi and j >= i:
                            j += 1
                        qi = q[b, kh * G, i]
                        k[b, kh, j] = 4.0 * qi / np.float32(np.linalg.norm(qi.astype(np.float64)))
        if w.sink:
            k[:, :, 0, :] *= 6.0
    elif w.values != "iid":
        raise ValueError(w.values)
    if v_ones:
        v = np.ones_like(v)
    qb, qf = to_16bit(q, w.dtype)
    del q
    kb, kf = to_16bit(k, w.dtype)
    del k
    vb, vf = to_16bit(v, w.dtype)
    del v
    return Tensors(qb, kb, vb, qf, kf, vf)


def sample_rows(w: Workload, n_per_head: int, seed: Optional[int] = None) -> np.ndarray:
    """Seeded query-row sample, one sorted row list per (batch, head): int64 [B, H, n]."""
    rng = np.random.Generator(np.random.PCG64(w.seed + 7 if seed is None else seed))
    n = min(n_per_head, w.Lq)
    out = np.empty((w.B, w.H, n), dtype=np.int64)
    for b in range(w.B):
        for h in range(w.H):
            out[b, h] = np.sort(rng.choice(w.Lq, size=n, replace=False))
    return out


def sample_tiles(w: Workload, n_per_head: int, seed: Optional[int] = None) -> np.ndarray:
    """Seeded query-tile sample per (batch, head): int64 [B, H, n] tile indices."""
    rng = np.random.Generator(np.random.PCG64(w.seed + 11 if seed is None else seed))
    n = min(n_per_head, w.nqt)
    out = np.empty((w.B, w.H, n), dtype=np.int64)
    for b in range(w.B):
        for h in range(w.H):
            out[b, h] = np.sort(rng.choice(w.nqt, size=n, replace=False))
    return out


def tflop(w: Workload) -> float:
    return w.flops() / 1e12


__all__ = ["Workload", "CONFIGS", "config_by_name", "make_workload", "sample_rows",
           "sample_tiles", "to_16bit", "bf16_bits_to_f32", "Tensors", "tflop"]
