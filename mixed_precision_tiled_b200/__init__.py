"""Tile-routed mixed-precision prefill attention for B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/lamp.h`` (library
``mixed_precision_tiled_b200/_build/liblamp.so``).  Every function below only marshals
arguments (torch tensors or integer device pointers -> raw pointers, the current CUDA stream)
and raises ``LampError`` on a non-zero status; all computation runs in the library's CUDA
kernels.  There is no CPU path: if the library is missing, importing the first entry point
fails loudly.

The method (TileMix page, section 2; LampAttention abstract): Q and K are quantised per block
to 8 bits; QK^T score tiles are computed in 8 bits, except tiles routed to 16 bits by a packed
per-query-tile bitmask (one bit per group of key tiles, 0 = FP16) or flagged by the look-ahead
rule (8-bit tile max within tau of the running row max); both feed one online softmax and a
16-bit P.V.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_build", "liblamp.so")

LAMP_OK, LAMP_ERR_INVALID, LAMP_ERR_UNSUPPORTED, LAMP_ERR_CUDA, LAMP_ERR_TIMEOUT = range(5)
ROUTE_BITMASK, ROUTE_ADAPTIVE = 0x0, 0x1
FMT_INT8, FMT_E4M3 = 0x0, 0x2
IN_FP16, IN_BF16 = 0x0, 0x4
OUT_F32, OUT_INDTYPE = 0x0, 0x8
PV_E4M3 = 0x10  # 8-bit exponentials and an 8-bit P.V

EXPORTS = ("lamp_tile_shape", "lamp_mask_words", "lamp_quant_qk", "lamp_build_mask",
           "lamp_build_mask_template", "lamp_template_fraction",
           "lamp_template_for_int8_fraction", "lamp_quant_qk_varlen", "lamp_attn_fwd_q8_varlen", "lamp_attn_fwd_q8_skip", "lamp_decode_fwd",
           "lamp_attn_fwd_varlen", "lamp_attn_fwd", "lamp_attn_fwd_q8", "lamp_attn_fwd_noalloc", "lamp_attn_fwd_host",
           "lamp_quant_v", "lamp_attn_fwd_q8_pv8",
           "lamp_workspace_size",
           "lamp_set_workspace", "lamp_check", "lamp_selftest_timeout", "lamp_mma_probe",
           "lamp_attn_debug", "lamp_exp2_eval", "lamp_last_error")
NOALLOC_MAX_BYTES = 32 << 20  # LAMP_NOALLOC_MAX_BYTES


class LampError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"lamp error {code}: {msg}")
        self.code = code


_lib = None
_lock = threading.Lock()
_vp, _i, _f, _u64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64, ctypes.c_size_t


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: run `python -m mixed_precision_tiled_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            sig = {
                "lamp_tile_shape": (_i, [_i, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
                "lamp_mask_words": (_i, [_i, _i, _i]),
                "lamp_quant_qk": (_i, [_vp, _vp, _vp, _vp, _vp, _vp] + [_i] * 7 + [_vp]),
                "lamp_build_mask": (_i, [_vp] + [_i] * 6 + [_f, _u64, _vp]),
                "lamp_build_mask_template": (_i, [_vp] + [_i] * 9 + [_vp]),
                "lamp_template_fraction": (_i, [_i] * 9 + [ctypes.POINTER(ctypes.c_double)]),
                "lamp_template_for_int8_fraction": (_i, [_i] * 6 + [ctypes.c_double]
                                                    + [ctypes.POINTER(_i)] * 3
                                                    + [ctypes.POINTER(ctypes.c_double)]),
                "lamp_attn_fwd": (_i, [_vp] * 5 + [_i] * 8 + [_f, _vp, _i, _i, _f, _vp]),
                "lamp_quant_qk_varlen": (_i, [_vp] * 8 + [_i] * 9 + [_vp]),
                "lamp_attn_fwd_q8_skip": (_i, [_vp] * 9 + [_i] * 8 + [_f, _i, _f, _f, _vp, _vp]),
                "lamp_decode_fwd": (_i, [_vp] * 10 + [_i] * 5 + [_f, _vp, _i, _i, _vp]),
                "lamp_attn_fwd_q8_varlen": (_i, [_vp] * 11 + [_i] * 10 + [_f, _vp, _i, _i, _f, _vp, _vp]),
                "lamp_attn_fwd_varlen": (_i, [_vp] * 7 + [_i] * 10 + [_f, _vp, _i, _i, _f, _vp]),
                "lamp_attn_fwd_q8": (_i, [_vp] * 9 + [_i] * 8 + [_f, _vp, _i, _i, _f, _vp, _vp]),
                "lamp_attn_fwd_noalloc": (_i, [_vp] * 5 + [_i] * 8 + [_f, _vp, _i, _i, _f, _vp]),
                "lamp_attn_fwd_host": (_i, [_vp] * 5 + [_i] * 8 + [_f, _vp, _i, _i, _f, _i, _vp]),
                "lamp_quant_v": (_i, [_vp] * 3 + [_i] * 5 + [_vp]),
                "lamp_attn_fwd_q8_pv8": (_i, [_vp] * 10 + [_i] * 8 + [_f, _vp, _i, _i, _f, _vp]),
                "lamp_workspace_size": (_sz, [_i] * 7),
                "lamp_set_workspace": (_i, [_vp, _sz]),
                "lamp_check": (_i, [_vp]),
                "lamp_selftest_timeout": (_i, [_u64, _vp]),
                "lamp_mma_probe": (_i, [_i, _i, _i, _vp]),
                "lamp_attn_debug": (_i, [_vp] * 9 + [_i] * 8 + [_f, _vp, _i, _i, _f, _vp, _vp, _i,
                                                            _vp, _vp, _vp]),
                "lamp_exp2_eval": (_i, [_vp, _vp, _i, _i, _vp]),
                "lamp_last_error": (ctypes.c_char_p, []),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype, fn.argtypes = res, args
            _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int):
    if code != LAMP_OK:
        raise LampError(code, lib().lamp_last_error().decode())


def mode_bits(route="bitmask", fmt="int8", dtype="bf16", out="f32", pv8=False) -> int:
    return ((ROUTE_ADAPTIVE if route == "adaptive" else ROUTE_BITMASK)
            | (FMT_E4M3 if fmt == "e4m3" else FMT_INT8)
            | (IN_BF16 if dtype == "bf16" else IN_FP16)
            | (OUT_INDTYPE if out == "in" else OUT_F32)
            | (PV_E4M3 if pv8 else 0))


# ------------------------------------------------------------ C-ABI wrappers ----------

def lamp_tile_shape(D: int):
    bm, bn = _i(), _i()
    _check(lib().lamp_tile_shape(D, ctypes.byref(bm), ctypes.byref(bn)))
    return bm.value, bn.value


def lamp_mask_words(Lk: int, D: int, group_tiles: int) -> int:
    w = lib().lamp_mask_words(Lk, D, group_tiles)
    if w < 0:
        raise LampError(LAMP_ERR_INVALID, "invalid arguments to lamp_mask_words")
    return w


def lamp_quant_qk(q, k, q8, k8, q_scale, k_scale, B, H, Hkv, Lq, Lk, D, mode, stream=None):
    _check(lib().lamp_quant_qk(_ptr(q), _ptr(k), _ptr(q8), _ptr(k8), _ptr(q_scale), _ptr(k_scale),
                               B, H, Hkv, Lq, Lk, D, mode, _stream(stream)))


def lamp_build_mask(mask_bits, B, H, Lq, Lk, D, group_tiles, fp16_fraction, seed, stream=None):
    _check(lib().lamp_build_mask(_ptr(mask_bits), B, H, Lq, Lk, D, group_tiles,
                                 float(fp16_fraction), int(seed) & (2**64 - 1), _stream(stream)))


def lamp_build_mask_template(mask_bits, B, H, Lq, Lk, D, group_tiles, sink_groups, band_groups,
                             stride_groups, stream=None):
    _check(lib().lamp_build_mask_template(_ptr(mask_bits), B, H, Lq, Lk, D, group_tiles,
                                          sink_groups, band_groups, stride_groups,
                                          _stream(stream)))


def lamp_template_fraction(Lq, Lk, D, group_tiles, causal, window, sink_groups, band_groups,
                           stride_groups) -> float:
    out = ctypes.c_double()
    _check(lib().lamp_template_fraction(Lq, Lk, D, group_tiles, int(causal), window, sink_groups,
                                        band_groups, stride_groups, ctypes.byref(out)))
    return out.value


def lamp_template_for_int8_fraction(Lq, Lk, D, group_tiles, causal, window, int8_fraction):
    """(sink_groups, band_groups, stride_groups, realised fp16 fraction)."""
    s, b, st, fr = _i(), _i(), _i(), ctypes.c_double()
    _check(lib().lamp_template_for_int8_fraction(Lq, Lk, D, group_tiles, int(causal), window,
                                                 float(int8_fraction), ctypes.byref(s),
                                                 ctypes.byref(b), ctypes.byref(st),
                                                 ctypes.byref(fr)))
    return s.value, b.value, st.value, fr.value


def lamp_attn_fwd_q8_skip(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D,
                          causal, window, scale, mode, tau, skip_tau, route_out=None,
                          stream=None):
    _check(lib().lamp_attn_fwd_q8_skip(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8),
                                       _ptr(q_scale), _ptr(k_scale), _ptr(o), _ptr(lse), B, H,
                                       Hkv, Lq, Lk, D, int(causal), window, float(scale), mode,
                                       float(tau), float(skip_tau), _ptr(route_out),
                                       _stream(stream)))


def lamp_decode_fwd(q, q8, q_scale, k8, k_scale, v8, v_scale, len_k, o, lse, B, H, Hkv, max_k,
                    D, scale, mask_bits, group_tiles, mode, stream=None):
    _check(lib().lamp_decode_fwd(_ptr(q), _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale),
                                 _ptr(v8), _ptr(v_scale), _ptr(len_k), _ptr(o), _ptr(lse), B, H,
                                 Hkv, max_k, D, float(scale), _ptr(mask_bits), group_tiles, mode,
                                 _stream(stream)))


def lamp_quant_qk_varlen(q, k, q8, k8, q_scale, k_scale, cu_q, cu_k, B, H, Hkv, max_q, max_k,
                         total_q, total_k, D, mode, stream=None):
    _check(lib().lamp_quant_qk_varlen(_ptr(q), _ptr(k), _ptr(q8), _ptr(k8), _ptr(q_scale),
                                      _ptr(k_scale), _ptr(cu_q), _ptr(cu_k), B, H, Hkv, max_q,
                                      max_k, total_q, total_k, D, mode, _stream(stream)))


def lamp_attn_fwd_q8_varlen(q, k, v, q8, k8, q_scale, k_scale, o, lse, cu_q, cu_k, B, H, Hkv,
                            max_q, max_k, total_q, total_k, D, causal, window, scale, mask_bits,
                            group_tiles, mode, tau, route_out=None, stream=None):
    _check(lib().lamp_attn_fwd_q8_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8),
                                         _ptr(q_scale), _ptr(k_scale), _ptr(o), _ptr(lse),
                                         _ptr(cu_q), _ptr(cu_k), B, H, Hkv, max_q, max_k, total_q,
                                         total_k, D, int(causal), window, float(scale),
                                         _ptr(mask_bits), group_tiles, mode, float(tau),
                                         _ptr(route_out), _stream(stream)))


def lamp_attn_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, Hkv, max_q, max_k, total_q, total_k,
                         D, causal, window, scale, mask_bits, group_tiles, mode, tau,
                         stream=None):
    _check(lib().lamp_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_q),
                                      _ptr(cu_k), B, H, Hkv, max_q, max_k, total_q, total_k, D,
                                      int(causal), window, float(scale), _ptr(mask_bits),
                                      group_tiles, mode, float(tau), _stream(stream)))


def lamp_attn_fwd(q, k, v, o, lse, B, H, Hkv, Lq, Lk, D, causal, window, scale, mask_bits,
                  group_tiles, mode, tau, stream=None):
    _check(lib().lamp_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Lq, Lk,
                               D, int(causal), int(window), float(scale), _ptr(mask_bits),
                               int(group_tiles), int(mode), float(tau), _stream(stream)))


def lamp_attn_fwd_noalloc(q, k, v, o, lse, B, H, Hkv, Lq, Lk, D, causal, window, scale,
                          mask_bits, group_tiles, mode, tau, stream=None):
    """lamp_attn_fwd without any device allocation (scratch in a fixed device array)."""
    _check(lib().lamp_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv,
                                       Lq, Lk, D, int(causal), int(window), float(scale),
                                       _ptr(mask_bits), int(group_tiles), int(mode), float(tau),
                                       _stream(stream)))


def lamp_attn_fwd_host(q, k, v, o, lse, B, H, Hkv, Lq, Lk, D, causal, window, scale, mask_bits,
                       group_tiles, mode, tau, n_chunks=0, stream=None):
    """lamp_attn_fwd on host buffers (q, k, v, o, lse: pinned CPU tensors or host addresses),
    the copies pipelined against the compute; mask_bits stays on the device."""
    _check(lib().lamp_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Lq,
                                    Lk, D, int(causal), int(window), float(scale),
                                    _ptr(mask_bits), int(group_tiles), int(mode), float(tau),
                                    int(n_chunks), _stream(stream)))


def lamp_quant_v(v, v8t, v_scale, B, Hkv, Lk, D, mode, stream=None):
    _check(lib().lamp_quant_v(_ptr(v), _ptr(v8t), _ptr(v_scale), B, Hkv, Lk, D, int(mode),
                              _stream(stream)))


def lamp_attn_fwd_q8_pv8(q, k, q8, k8, q_scale, k_scale, v8t, v_scale, o, lse, B, H, Hkv, Lq, Lk,
                         D, causal, window, scale, mask_bits, group_tiles, mode, tau, stream=None):
    _check(lib().lamp_attn_fwd_q8_pv8(_ptr(q), _ptr(k), _ptr(q8), _ptr(k8), _ptr(q_scale),
                                      _ptr(k_scale), _ptr(v8t), _ptr(v_scale), _ptr(o), _ptr(lse),
                                      B, H, Hkv, Lq, Lk, D, int(causal), int(window), float(scale),
                                      _ptr(mask_bits), int(group_tiles), int(mode), float(tau),
                                      _stream(stream)))


def lamp_attn_fwd_q8(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                     window, scale, mask_bits, group_tiles, mode, tau, route_out=None,
                     stream=None):
    _check(lib().lamp_attn_fwd_q8(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(q_scale),
                                  _ptr(k_scale), _ptr(o), _ptr(lse), B, H, Hkv, Lq, Lk, D,
                                  int(causal), int(window), float(scale), _ptr(mask_bits),
                                  int(group_tiles), int(mode), float(tau), _ptr(route_out),
                                  _stream(stream)))


def lamp_attn_debug(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                    window, scale, mask_bits, group_tiles, mode, tau, route_out, tile_slot,
                    n_slots, s8_dump, s16_dump, stream=None):
    _check(lib().lamp_attn_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(q_scale),
                                 _ptr(k_scale), _ptr(o), _ptr(lse), B, H, Hkv, Lq, Lk, D,
                                 int(causal), int(window), float(scale), _ptr(mask_bits),
                                 int(group_tiles), int(mode), float(tau), _ptr(route_out),
                                 _ptr(tile_slot), int(n_slots), _ptr(s8_dump), _ptr(s16_dump),
                                 _stream(stream)))


def lamp_exp2_eval(x, y, n, method, stream=None):
    _check(lib().lamp_exp2_eval(_ptr(x), _ptr(y), int(n), int(method), _stream(stream)))


def lamp_workspace_size(B, H, Hkv, Lq, Lk, D, mode=0) -> int:
    return int(lib().lamp_workspace_size(B, H, Hkv, Lq, Lk, D, mode))


def lamp_set_workspace(ptr, nbytes: int):
    _check(lib().lamp_set_workspace(_ptr(ptr), int(nbytes)))


def lamp_check(stream=None):
    _check(lib().lamp_check(_stream(stream)))


def lamp_mma_probe(kind: int, n: int, iters: int, stream=None):
    _check(lib().lamp_mma_probe(int(kind), int(n), int(iters), _stream(stream)))


def lamp_selftest_timeout(wait_ns: int, stream=None):
    _check(lib().lamp_selftest_timeout(int(wait_ns), _stream(stream)))


def lamp_last_error() -> str:
    return lib().lamp_last_error().decode()


# ------------------------------------------------------------ torch conveniences ------
# Allocation of outputs with torch (device memory is PyTorch's job here); the arithmetic
# stays in the library.

def attention(q, k, v, *, causal=False, window=0, scale=0.0, mask_bits=None, group_tiles=1,
              route="bitmask", fmt="int8", tau=0.0, out="f32", pv8=False, stream=None):
    """O, lse for q [B,H,Lq,D], k/v [B,Hkv,Lk,D] (fp16/bf16 CUDA tensors); ``pv8``: 8-bit
    exponentials and an 8-bit P.V (D = 128)."""
    import torch
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    dtype = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    o = torch.empty((B, H, Lq, D), device=q.device,
                    dtype=torch.float32 if out == "f32" else q.dtype)
    lse = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    lamp_attn_fwd(q, k, v, o, lse, B, H, Hkv, Lq, Lk, D, causal, window, scale, mask_bits,
                  group_tiles, mode_bits(route, fmt, dtype, out, pv8), tau, stream)
    return o, lse


def quantize_v(v, *, stream=None):
    """(v8t uint8 [B,Hkv,D,Lk16] channel-major E4M3 codes, v_scale float32 [B,Hkv,D]) for v
    [B,Hkv,Lk,D]; Lk16 = Lk rounded up to 16."""
    import torch
    B, Hkv, Lk, D = v.shape
    v8t = torch.empty((B, Hkv, D, (Lk + 15) // 16 * 16), device=v.device, dtype=torch.uint8)
    vs = torch.empty((B, Hkv, D), device=v.device, dtype=torch.float32)
    dtype = "bf16" if v.dtype == torch.bfloat16 else "fp16"
    lamp_quant_v(v, v8t, vs, B, Hkv, Lk, D, mode_bits(dtype=dtype), stream)
    return v8t, vs


def attention_q8_pv8(q, k, q8, k8, q_scale, k_scale, v8t, v_scale, *, causal=False, window=0,
                     scale=0.0, mask_bits=None, group_tiles=1, route="bitmask", fmt="int8",
                     tau=0.0, out="f32", stream=None):
    """The 8-bit P.V kernel alone on quantised Q, K (``quantize``) and V (``quantize_v``)."""
    import torch
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    dtype = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    o = torch.empty((B, H, Lq, D), device=q.device,
                    dtype=torch.float32 if out == "f32" else q.dtype)
    lse = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    lamp_attn_fwd_q8_pv8(q, k, q8, k8, q_scale, k_scale, v8t, v_scale, o, lse, B, H, Hkv, Lq, Lk,
                         D, causal, window, scale, mask_bits, group_tiles,
                         mode_bits(route, fmt, dtype, out, True), tau, stream)
    return o, lse


def quantize(q, k, *, fmt="int8", stream=None):
    """(q8, k8, q_scale, k_scale) for q [B,H,Lq,D], k [B,Hkv,Lk,D]."""
    import torch
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    bm, bn = lamp_tile_shape(D)
    q8 = torch.empty(q.shape, device=q.device, dtype=torch.uint8)
    k8 = torch.empty(k.shape, device=k.device, dtype=torch.uint8)
    qs = torch.empty((B, H, -(-Lq // bm)), device=q.device, dtype=torch.float32)
    ks = torch.empty((B, Hkv, -(-Lk // bn)), device=q.device, dtype=torch.float32)
    dtype = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    lamp_quant_qk(q, k, q8, k8, qs, ks, B, H, Hkv, Lq, Lk, D, mode_bits(fmt=fmt, dtype=dtype),
                  stream)
    return q8, k8, qs, ks


def build_mask(B, H, Lq, Lk, D, group_tiles, fp16_fraction, seed, device="cuda", stream=None):
    import torch
    bm, _ = lamp_tile_shape(D)
    W = lamp_mask_words(Lk, D, group_tiles)
    m = torch.empty((B, H, -(-Lq // bm), W), device=device, dtype=torch.int64)
    lamp_build_mask(m, B, H, Lq, Lk, D, group_tiles, fp16_fraction, seed, stream)
    return m


def build_mask_template(B, H, Lq, Lk, D, group_tiles, sink_groups, band_groups, stride_groups,
                        device="cuda", stream=None):
    import torch
    bm, _ = lamp_tile_shape(D)
    W = lamp_mask_words(Lk, D, group_tiles)
    m = torch.empty((B, H, -(-Lq // bm), W), device=device, dtype=torch.int64)
    lamp_build_mask_template(m, B, H, Lq, Lk, D, group_tiles, sink_groups, band_groups,
                             stride_groups, stream)
    return m


def attention_q8(q, k, v, q8, k8, q_scale, k_scale, *, causal=False, window=0, scale=0.0,
                 mask_bits=None, group_tiles=1, route="bitmask", fmt="int8", tau=0.0,
                 out="f32", want_route=False, skip_tau=None, stream=None):
    import torch
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    bm, bn = lamp_tile_shape(D)
    dtype = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    o = torch.empty((B, H, Lq, D), device=q.device,
                    dtype=torch.float32 if out == "f32" else q.dtype)
    lse = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    rmap = (torch.empty((B, H, -(-Lq // bm), -(-Lk // bn)), device=q.device, dtype=torch.uint8)
            if want_route else None)
    mode = mode_bits(route, fmt, dtype, out)
    if skip_tau is not None:
        lamp_attn_fwd_q8_skip(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D,
                              causal, window, scale, mode, tau, skip_tau, rmap, stream)
    else:
        lamp_attn_fwd_q8(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                         window, scale, mask_bits, group_tiles, mode, tau, rmap, stream)
    return (o, lse, rmap) if want_route else (o, lse)


def attention_debug(q, k, v, q8, k8, q_scale, k_scale, tiles, *, causal=False, window=0,
                    scale=0.0, mask_bits=None, group_tiles=1, route="bitmask", fmt="int8",
                    tau=0.0, stream=None):
    """lamp_attn_debug on torch tensors: ``tiles`` lists routing tiles (b, h, qt, kt).  Returns
    (o, lse, route map, s8 [n][BM][BN] int32 words, s16 [n][BM][BN] fp32); slots the kernel did
    not write keep the fill value 0x7fbadbad (int32) / NaN (fp32)."""
    import torch
    B, H, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    bm, bn = lamp_tile_shape(D)
    nqt, nkt = -(-Lq // bm), -(-Lk // bn)
    dtype = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    slot = torch.full((B, H, nqt, nkt), -1, dtype=torch.int32)
    for s_, (b, h, qt, kt) in enumerate(tiles):
        slot[b, h, qt, kt] = s_
    slot = slot.to(q.device)
    n = len(tiles)
    s8 = torch.full((n, bm, bn), 0x7FBADBAD, dtype=torch.int32, device=q.device)
    s16 = torch.full((n, bm, bn), float("nan"), dtype=torch.float32, device=q.device)
    o = torch.empty((B, H, Lq, D), device=q.device, dtype=torch.float32)
    lse = torch.empty((B, H, Lq), device=q.device, dtype=torch.float32)
    rmap = torch.empty((B, H, nqt, nkt), device=q.device, dtype=torch.uint8)
    lamp_attn_debug(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                    window, scale, mask_bits, group_tiles, mode_bits(route, fmt, dtype), tau,
                    rmap, slot, n, s8, s16, stream)
    return o, lse, rmap, s8, s16


def exp2_eval(x, method: int, stream=None):
    """The kernels' 2^x (method 0 polynomial, 1 hardware) on a float32 CUDA tensor."""
    import torch
    x = x.contiguous()
    y = torch.empty_like(x)
    lamp_exp2_eval(x, y, x.numel(), method, stream)
    return y
