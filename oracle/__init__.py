"""CPU oracle for tile-routed mixed-precision prefill attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
this package.  It shares no code with the CUDA library: the arithmetic lives in
``oracle.cpp`` (plain C++17 loops, fp64 softmax, exact integer / exact fp64 8-bit dot
products), built here with g++ and called through ctypes on numpy arrays.

What it computes, with the pages' passages it follows:
  * ``quantize``      -- per-block INT8 / E4M3 quantisation (TileMix page, section 2, "The
                         Dual-Path Engine", item 2; LampAttention abstract, "8-bit formats").
  * ``build_mask``    -- the packed routing bitmask, one bit per group of key tiles, 0 = FP16,
                         1 = INT8 (TileMix page, section 2, "Packed Bitmasks").
  * ``build_mask_template`` -- the structured static routing template (TileMix page, section
                         4, "static, data-free structured templates"; section 3, "SpTrans75").
  * ``attention``     -- routed scores, shared softmax and 16-bit-routed tiles (TileMix page,
                         section 2, "The Dual-Path Engine"; LampAttention abstract for the
                         adaptive 8-bit -> 16-bit recomputation, and, with ``pv8``, for
                         exponentials and P.V in 8-bit formats).
  * ``quantize_v``, ``e4m3_round_pos`` -- the 8-bit V and the rounding of the 8-bit p.
Every function is pinned by CPU tests against closed forms, brute force and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
            "-pthread"]


def build(force: bool = False) -> str:
    """Compile oracle.cpp into oracle/_build/liboracle.so (g++)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("Hkv", ctypes.c_int), ("Lq", ctypes.c_int),
        ("Lk", ctypes.c_int), ("D", ctypes.c_int), ("bm", ctypes.c_int), ("bn", ctypes.c_int),
        ("causal", ctypes.c_int), ("window", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("mask", ctypes.c_void_p), ("mask_words", ctypes.c_int), ("group_tiles", ctypes.c_int),
        ("adaptive", ctypes.c_int), ("fmt", ctypes.c_int), ("tau", ctypes.c_double),
        ("rows", ctypes.c_void_p), ("nrows", ctypes.c_int), ("threads", ctypes.c_int),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("route", ctypes.c_void_p),
        ("margin", ctypes.c_void_p), ("route_hint", ctypes.c_void_p),
        ("hint_margin", ctypes.c_double),
        ("q_codes", ctypes.c_void_p), ("q_scales", ctypes.c_void_p),
        ("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
        ("skip_tau", ctypes.c_double),
        ("k_codes_in", ctypes.c_void_p), ("k_scales_in", ctypes.c_void_p),
        ("hinted", ctypes.c_void_p),
        ("pv8", ctypes.c_int), ("v_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
        ("pv8_margin", ctypes.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            L.orc_e4m3_decode.restype = ctypes.c_double
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_encode.argtypes = [ctypes.c_float]
            L.orc_splitmix64_next.restype = ctypes.c_uint64
            L.orc_splitmix64_next.argtypes = [ctypes.c_uint64]
            L.orc_quantize.restype = None
            L.orc_quantize.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                       ctypes.c_void_p]
            L.orc_build_mask.restype = None
            L.orc_build_mask.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_uint64]
            L.orc_build_mask_template.restype = None
            L.orc_build_mask_template.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 10
            L.orc_attention.restype = ctypes.c_int
            L.orc_attention.argtypes = [ctypes.POINTER(_Args)]
            L.orc_e4m3_round_pos.restype = ctypes.c_double
            L.orc_e4m3_round_pos.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_double)]
            L.orc_quantize_v.restype = None
            L.orc_quantize_v.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
            L.orc_score_tiles.restype = ctypes.c_int
            L.orc_score_tiles.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 9 \
                + [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
            _lib = L
    return _lib


FMT = {"int8": 0, "e4m3": 1}


def _ptr(a):
    return None if a is None else a.ctypes.data


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    return int(lib().orc_e4m3_encode(float(x)))


def e4m3_round_pos(p: float):
    """(nearest e4m3 value of p >= 0, relative distance of p from the nearest rounding
    midpoint) -- the rounding of the 8-bit exponentials."""
    d = ctypes.c_double()
    r = lib().orc_e4m3_round_pos(float(p), ctypes.byref(d))
    return r, d.value


def quantize_v(x: np.ndarray):
    """Per-channel E4M3 V of x [..., Lk, D] (one scale per leading index and channel over all
    keys; LampAttention abstract, 8-bit formats, read for V).  Returns (codes uint8
    [..., D, Lk] channel-major, scales float32 [..., D])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    *lead, L, D = x.shape
    outer = int(np.prod(lead)) if lead else 1
    codes = np.empty((*lead, D, L), dtype=np.uint8)
    scales = np.empty((*lead, D), dtype=np.float32)
    lib().orc_quantize_v(_ptr(x), outer, L, D, _ptr(codes), _ptr(scales))
    return codes, scales


def splitmix64_next(state: int) -> int:
    return int(lib().orc_splitmix64_next(int(state) & 0xFFFFFFFFFFFFFFFF))


def quantize(x: np.ndarray, blk: int, fmt: str = "int8"):
    """Per-block quantisation of x [..., L, D] (fp32 values) in blocks of ``blk`` rows.

    Returns (codes uint8 [..., L, D] -- int8 two's complement or e4m3 bits --,
    scales float32 [..., ceil(L/blk)]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    *lead, L, D = x.shape
    outer = int(np.prod(lead)) if lead else 1
    nb = -(-L // blk)
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty((*lead, nb), dtype=np.float32)
    lib().orc_quantize(_ptr(x), outer, L, D, blk, FMT[fmt], _ptr(codes), _ptr(scales))
    return codes, scales


def mask_words(nkt: int, group_tiles: int) -> int:
    ng = -(-nkt // group_tiles)
    return max(1, -(-ng // 64))


def build_mask(B: int, H: int, nqt: int, nkt: int, group_tiles: int, p_fp16: float,
               seed: int) -> np.ndarray:
    """uint64 [B, H, nQT, W] routing mask drawn from the seeded SplitMix64 template."""
    ng = -(-nkt // group_tiles)
    W = mask_words(nkt, group_tiles)
    m = np.empty((B, H, nqt, W), dtype=np.uint64)
    lib().orc_build_mask(_ptr(m), B, H, nqt, ng, W, float(p_fp16), int(seed) & (2**64 - 1))
    return m


def build_mask_template(B: int, H: int, Lq: int, Lk: int, bm: int, bn: int, group_tiles: int,
                        sink: int, band: int, stride: int) -> np.ndarray:
    """uint64 [B, H, nQT, W] structured static routing template (TileMix page, section 4,
    "static, data-free structured templates"; section 3, the 75%-INT8 "SpTrans75"
    configuration): group g of routing row qt is FP16 iff g < sink, |gd - g| < band, or stride
    divides |gd - g|, gd being the group of the key aligned with the row's last query."""
    nqt, nkt = -(-Lq // bm), -(-Lk // bn)
    W = mask_words(nkt, group_tiles)
    m = np.empty((B, H, nqt, W), dtype=np.uint64)
    lib().orc_build_mask_template(_ptr(m), B, H, Lq, Lk, bm, bn, group_tiles, int(sink),
                                  int(band), int(stride))
    return m


def attention(q, k, v, *, bm, bn, causal=False, window=0, scale=None, mask=None, group_tiles=1,
              route="bitmask", fmt="int8", tau=0.0, rows=None, threads=0, want_codes=False,
              route_hint=None, hint_margin=0.0, skip_tau=float("inf"), k_codes_in=None,
              k_scales_in=None, pv8=False):
    """Routed attention on fp32 values of 16-bit inputs.

    q [B,H,Lq,D], k/v [B,Hkv,Lk,D].  ``mask`` uint64 [B,H,nQT,W] or None (all 8-bit) in
    bitmask routing.  ``rows`` int64 [B,H,n] (sorted per head) restricts the output rows.
    Returns a dict with o (fp64 [B,H,R,D]), lse (fp64 [B,H,R]), route (uint8 [B,H,nQT,nKT]:
    0 dead, 1 8-bit, 2 16-bit by mask, 3 16-bit flagged, 4 dropped), margin (fp64, adaptive
    decisions), hinted (uint8, 1 where a decision followed ``route_hint`` against the rule's
    own outcome, which only happens where its margin is below ``hint_margin``).  ``k_codes_in`` / ``k_scales_in`` (uint8 [B,Hkv,Lk,D], float32 [B,Hkv,nKT]):
    an 8-bit key cache used by the 8-bit path instead of quantising ``k`` (decode with an INT8
    KV cache: TileMix page, section 4).  ``skip_tau`` (look-ahead mode; LATTE page, low-precision filtering of the keys
    far below the row maximum, read per tile): a tile every row of which has t_r < m_r -
    skip_tau is dropped; +inf never drops.  ``pv8``: 8-bit exponentials and an 8-bit P.V
    (LampAttention abstract): V in per-channel E4M3 (``quantize_v``), each p = e^(s - m_t)
    * 2^8 rounded to E4M3 against the running max m_t after its key tile (ascending tiles), O =
    sv * sum p8 v8 / sum p8 over the tiles rescaled to the final max; adds v_codes, v_scales and
    pv8_margin (per output row, the smallest relative distance of one of its p from an E4M3
    rounding midpoint).  lse stays the exact softmax's.
    """
    q = np.ascontiguousarray(q, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    nqt, nkt = -(-Lq // bm), -(-Lk // bn)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = rows.shape[-1]
    else:
        R = Lq
    o = np.empty((B, H, R, D), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    rmap = np.empty((B, H, nqt, nkt), dtype=np.uint8)
    margin = np.empty((B, H, nqt, nkt), dtype=np.float64)
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint64)
    if route_hint is not None:
        route_hint = np.ascontiguousarray(route_hint, dtype=np.uint8)
    a = _Args()
    a.q, a.k, a.v = _ptr(q), _ptr(k), _ptr(v)
    a.B, a.H, a.Hkv, a.Lq, a.Lk, a.D, a.bm, a.bn = B, H, Hkv, Lq, Lk, D, bm, bn
    a.causal, a.window = int(bool(causal)), int(window)
    a.scale = float(scale)
    a.mask = _ptr(mask)
    a.mask_words = mask.shape[-1] if mask is not None else 0
    a.group_tiles = int(group_tiles)
    a.adaptive = 1 if route == "adaptive" else 0
    a.fmt = FMT[fmt]
    a.tau = float(tau)
    a.rows = _ptr(rows)
    a.nrows = R if rows is not None else 0
    a.threads = int(threads) if threads else (os.cpu_count() or 1)
    a.o, a.lse, a.route, a.margin = _ptr(o), _ptr(lse), _ptr(rmap), _ptr(margin)
    a.route_hint = _ptr(route_hint)
    a.hint_margin = float(hint_margin)
    a.skip_tau = float(skip_tau)
    if k_codes_in is not None:  # an 8-bit key cache: codes and scales given, not recomputed
        k_codes_in = np.ascontiguousarray(k_codes_in, dtype=np.uint8)
        k_scales_in = np.ascontiguousarray(k_scales_in, dtype=np.float32)
        assert k_codes_in.shape == k.shape and k_scales_in.shape == (B, Hkv, nkt)
        a.k_codes_in, a.k_scales_in = _ptr(k_codes_in), _ptr(k_scales_in)
    hinted = np.zeros((B, H, nqt, nkt), dtype=np.uint8)
    a.hinted = _ptr(hinted)
    out = {"o": o, "lse": lse, "route": rmap, "margin": margin, "hinted": hinted}
    if pv8:
        vcodes = np.empty((B, Hkv, D, Lk), np.uint8)
        vscales = np.empty((B, Hkv, D), np.float32)
        pmargin = np.empty((B, H, R), np.float64)
        a.pv8, a.v_codes, a.v_scales, a.pv8_margin = 1, _ptr(vcodes), _ptr(vscales), _ptr(pmargin)
        out.update(v_codes=vcodes, v_scales=vscales, pv8_margin=pmargin)
    if want_codes:
        qc = np.empty(q.shape, np.uint8)
        qs = np.empty((B, H, nqt), np.float32)
        kc = np.empty(k.shape, np.uint8)
        ks = np.empty((B, Hkv, nkt), np.float32)
        a.q_codes, a.q_scales, a.k_codes, a.k_scales = _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks)
        out.update(q_codes=qc, q_scales=qs, k_codes=kc, k_scales=ks)
    rc = lib().orc_attention(ctypes.byref(a))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out


def score_tiles(qx, kx, bm: int, bn: int, kind: str, tiles) -> np.ndarray:
    """Raw (unscaled) score tiles, the reference of the library's debug capture.

    ``tiles``: (b, h, qt, kt) routing tiles.  ``kind``: "int8" / "e4m3" (qx, kx uint8 codes
    [B,H,Lq,D] / [B,Hkv,Lk,D], exact sums of code products) or "16bit" (fp32 values of the
    16-bit inputs, fp64 sums).  Rows and keys past the problem count as zero vectors.  Returns
    fp64 [n, bm, bn] (the INT8 sums are integers, exact in fp64)."""
    kinds = {"int8": 0, "e4m3": 1, "16bit": 2}
    dt = np.float32 if kind == "16bit" else np.uint8
    qx = np.ascontiguousarray(qx, dtype=dt)
    kx = np.ascontiguousarray(kx, dtype=dt)
    B, H, Lq, D = qx.shape
    _, Hkv, Lk, _ = kx.shape
    t = np.ascontiguousarray(np.asarray(tiles, dtype=np.int32).reshape(-1, 4))
    out = np.empty((t.shape[0], bm, bn), dtype=np.float64)
    rc = lib().orc_score_tiles(_ptr(qx), _ptr(kx), B, H, Hkv, Lq, Lk, D, bm, bn, kinds[kind],
                               _ptr(t), t.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the tile list")
    return out
