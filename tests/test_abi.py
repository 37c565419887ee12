"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import mixed_precision_tiled_b200 as mpt
from mixed_precision_tiled_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    mbuild.build()


def header_functions():
    src = open(os.path.join(ROOT, "include", "lamp.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lamp_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 11
    out = subprocess.check_output(["nm", "-D", "--defined-only", mbuild.LIB]).decode()
    exported = set(re.findall(r" T (lamp_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(names) == set(mpt.EXPORTS)
    L = ctypes.CDLL(mbuild.LIB)
    for n in names:
        getattr(L, n)


def test_tile_shapes_and_mask_words():
    assert mpt.lamp_tile_shape(64) == (64, 64)
    assert mpt.lamp_tile_shape(128) == (128, 128)
    assert mpt.lamp_tile_shape(256) == (64, 128)
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_tile_shape(96)
    assert e.value.code == mpt.LAMP_ERR_UNSUPPORTED
    # config geometry: W = ceil(ceil(nKT / g) / 64)
    assert mpt.lamp_mask_words(4096, 128, 4) == 1
    assert mpt.lamp_mask_words(131072, 128, 8) == 2
    assert mpt.lamp_mask_words(65536, 128, 8) == 1
    assert mpt.lamp_mask_words(16384, 256, 2) == 1
    assert mpt.lamp_mask_words(8193, 128, 1) == 2   # 65 key tiles
    with pytest.raises(mpt.LampError):
        mpt.lamp_mask_words(0, 128, 1)


def _attn_args(**kw):
    a = dict(q=0x1000, k=0x2000, v=0x3000, o=0x4000, lse=0x5000, B=1, H=4, Hkv=2, Lq=128,
             Lk=128, D=128, causal=1, window=0, scale=0.0, mask_bits=None, group_tiles=1,
             mode=0, tau=0.0)
    a.update(kw)
    return a


@pytest.mark.parametrize("bad,code", [
    (dict(H=3, Hkv=2), mpt.LAMP_ERR_INVALID),
    (dict(B=0), mpt.LAMP_ERR_INVALID),
    (dict(Lq=0), mpt.LAMP_ERR_INVALID),
    (dict(D=80), mpt.LAMP_ERR_UNSUPPORTED),
    (dict(q=None), mpt.LAMP_ERR_INVALID),
    # the checks of the attention kernel itself also run before the quantiser is enqueued
    (dict(q=0x1001), mpt.LAMP_ERR_INVALID),
    (dict(o=0x5010), mpt.LAMP_ERR_INVALID),
    (dict(causal=0, window=16), mpt.LAMP_ERR_UNSUPPORTED),
    (dict(window=-1), mpt.LAMP_ERR_INVALID),
    (dict(group_tiles=0), mpt.LAMP_ERR_INVALID),
    (dict(mode=0x30), mpt.LAMP_ERR_INVALID),
    (dict(mode=1, tau=float("nan")), mpt.LAMP_ERR_INVALID),
    (dict(scale=float("nan")), mpt.LAMP_ERR_INVALID),
])
@pytest.mark.parametrize("entry", ["lamp_attn_fwd", "lamp_attn_fwd_noalloc"])
def test_attn_fwd_rejects_bad_arguments_on_host(bad, code, entry):
    with pytest.raises(mpt.LampError) as e:
        getattr(mpt, entry)(**_attn_args(**bad), stream=0)
    assert e.value.code == code


def test_pv8_entries_reject_bad_arguments_on_host():
    pv8 = mpt.mode_bits(pv8=True)
    a = _attn_args()
    args = lambda **kw: {**a, **kw}
    # the 8-bit P.V mode: D = 128, dense, no skip; the q8 entry points route it to the pv8 one
    for D, code in ((64, mpt.LAMP_ERR_UNSUPPORTED), (256, mpt.LAMP_ERR_UNSUPPORTED)):
        with pytest.raises(mpt.LampError) as e:
            mpt.lamp_attn_fwd(**args(D=D, mode=pv8), stream=0)
        assert e.value.code == code
    x = args(mode=pv8)
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_attn_fwd_q8(x["q"], x["k"], x["v"], 0x6000, 0x7000, 0x8000, 0x9000, x["o"],
                             x["lse"], x["B"], x["H"], x["Hkv"], x["Lq"], x["Lk"], x["D"],
                             x["causal"], x["window"], x["scale"], x["mask_bits"],
                             x["group_tiles"], x["mode"], x["tau"], None, stream=0)
    assert e.value.code == mpt.LAMP_ERR_UNSUPPORTED
    def q8pv8(**kw):
        y = args(**kw)
        mpt.lamp_attn_fwd_q8_pv8(y["q"], y["k"], 0x6000, 0x7000, 0x8000, 0x9000, y["v"],
                                 kw.get("v_scale", 0xA000), y["o"], y["lse"], y["B"], y["H"],
                                 y["Hkv"], y["Lq"], y["Lk"], y["D"], y["causal"], y["window"],
                                 y["scale"], y["mask_bits"], y["group_tiles"], y["mode"], y["tau"],
                                 stream=0)
    for kw, code in ((dict(mode=0), mpt.LAMP_ERR_INVALID),            # the bit is required
                     (dict(mode=pv8, v_scale=None), mpt.LAMP_ERR_INVALID),
                     (dict(mode=pv8, D=64), mpt.LAMP_ERR_UNSUPPORTED),
                     (dict(mode=pv8, v=0x1008), mpt.LAMP_ERR_INVALID)):  # V codes 16-byte aligned
        with pytest.raises(mpt.LampError) as e:
            q8pv8(**kw)
        assert e.value.code == code, kw
    for kw in (dict(v=None), dict(v8t=0x1008), dict(D=80), dict(Lk=0)):
        call = dict(v=0x1000, v8t=0x2000, v_scale=0x3000, B=1, Hkv=2, Lk=64, D=128, mode=0)
        call.update(kw)
        with pytest.raises(mpt.LampError):
            mpt.lamp_quant_v(call["v"], call["v8t"], call["v_scale"], call["B"], call["Hkv"],
                             call["Lk"], call["D"], call["mode"], stream=0)


@pytest.mark.parametrize("bad,code", [
    (dict(H=3, Hkv=2), mpt.LAMP_ERR_INVALID),
    (dict(B=0), mpt.LAMP_ERR_INVALID),
    (dict(D=80), mpt.LAMP_ERR_UNSUPPORTED),
    (dict(q=None), mpt.LAMP_ERR_INVALID),
    (dict(o=None), mpt.LAMP_ERR_INVALID),
    (dict(causal=0, window=16), mpt.LAMP_ERR_UNSUPPORTED),
    (dict(group_tiles=0), mpt.LAMP_ERR_INVALID),
    (dict(mode=0x30), mpt.LAMP_ERR_INVALID),
    (dict(scale=float("nan")), mpt.LAMP_ERR_INVALID),
    (dict(n_chunks=-1), mpt.LAMP_ERR_INVALID),
])
def test_attn_fwd_host_rejects_bad_arguments_on_host(bad, code):
    # host buffers need no alignment, so an odd host address alone is no error; everything else
    # lamp_attn_fwd checks is checked before anything is enqueued
    n_chunks = bad.pop("n_chunks", 0)
    a = _attn_args(**bad)
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_attn_fwd_host(**a, n_chunks=n_chunks, stream=0)
    assert e.value.code == code


@pytest.mark.parametrize("bad,code", [
    (dict(q=0x1001), mpt.LAMP_ERR_INVALID),            # misaligned
    (dict(o=0x5010), mpt.LAMP_ERR_INVALID),            # O written with 32-byte stores
    (dict(causal=0, window=16), mpt.LAMP_ERR_UNSUPPORTED),
    (dict(window=-1), mpt.LAMP_ERR_INVALID),
    (dict(group_tiles=0), mpt.LAMP_ERR_INVALID),
    (dict(mode=0x30), mpt.LAMP_ERR_INVALID),
    (dict(mode=1, tau=float("nan")), mpt.LAMP_ERR_INVALID),
])
def test_attn_fwd_q8_rejects_bad_arguments_on_host(bad, code):
    a = _attn_args(**bad)
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_attn_fwd_q8(a["q"], a["k"], a["v"], 0x6000, 0x7000, 0x8000, 0x9000, a["o"],
                             a["lse"], a["B"], a["H"], a["Hkv"], a["Lq"], a["Lk"], a["D"],
                             a["causal"], a["window"], a["scale"], a["mask_bits"],
                             a["group_tiles"], a["mode"], a["tau"], None, stream=0)
    assert e.value.code == code


def test_quant_and_mask_reject_bad_arguments_on_host():
    with pytest.raises(mpt.LampError):
        mpt.lamp_quant_qk(0x1000, None, 0x2000, None, None, None, 1, 1, 1, 64, 64, 64, 0, stream=0)
    with pytest.raises(mpt.LampError):
        mpt.lamp_quant_qk(0x1008, None, 0x2000, None, 0x3000, None, 1, 1, 1, 64, 64, 64, 0,
                          stream=0)
    with pytest.raises(mpt.LampError):
        mpt.lamp_build_mask(None, 1, 1, 64, 64, 64, 1, 0.5, 1, stream=0)
    with pytest.raises(mpt.LampError):
        mpt.lamp_build_mask(0x1000, 1, 1, 64, 64, 64, 1, 1.5, 1, stream=0)
    with pytest.raises(mpt.LampError):
        mpt.lamp_selftest_timeout(0, stream=0)


def test_workspace_size_and_alignment():
    n = mpt.lamp_workspace_size(1, 32, 8, 4096, 4096, 128)
    # q8 + k8 bytes plus the two scale arrays, each 256-byte aligned
    assert n == 32 * 4096 * 128 + 8 * 4096 * 128 + 32 * 32 * 4 + 8 * 32 * 4
    assert mpt.lamp_workspace_size(1, 1, 1, 1, 1, 96) == 0
    with pytest.raises(mpt.LampError):
        mpt.lamp_set_workspace(0x1010, 1024)
    mpt.lamp_set_workspace(None, 0)


@pytest.mark.parametrize("kind,n,iters", [(3, 128, 8), (-1, 128, 8), (0, 120, 8), (0, 272, 8),
                                          (1, 0, 8), (1, 192, 8), (2, 128, 0),
                                          (2, 128, (1 << 20) + 1)])
def test_mma_probe_rejects_bad_shapes_on_host(kind, n, iters):
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_mma_probe(kind, n, iters, stream=0)
    assert e.value.code == mpt.LAMP_ERR_INVALID


def test_template_calls_reject_bad_arguments_on_host():
    L = mpt.lib()
    d = ctypes.c_double()
    i1, i2, i3 = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    # (a non-null dummy pointer: the call must fail before any launch)
    assert L.lamp_build_mask_template(None, 1, 1, 256, 256, 64, 1, 0, 1, 0, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_build_mask_template(0x1000, 1, 1, 256, 256, 64, 1, -1, 1, 0, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_build_mask_template(0x1000, 1, 1, 256, 256, 64, 0, 0, 1, 0, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_build_mask_template(0x1000, 1, 1, 256, 256, 96, 1, 0, 1, 0, None) == mpt.LAMP_ERR_UNSUPPORTED
    assert L.lamp_template_fraction(256, 256, 64, 1, 1, 0, 0, 1, 0, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_template_fraction(256, 256, 64, 1, 0, 64, 0, 1, 0, ctypes.byref(d)) == mpt.LAMP_ERR_UNSUPPORTED
    assert L.lamp_template_fraction(0, 256, 64, 1, 1, 0, 0, 1, 0, ctypes.byref(d)) == mpt.LAMP_ERR_INVALID
    assert L.lamp_template_for_int8_fraction(256, 256, 64, 1, 1, 0, 1.5, ctypes.byref(i1),
                                             ctypes.byref(i2), ctypes.byref(i3),
                                             ctypes.byref(d)) == mpt.LAMP_ERR_INVALID
    assert L.lamp_template_for_int8_fraction(256, 256, 64, 1, 1, 0, 0.75, None, ctypes.byref(i2),
                                             ctypes.byref(i3), ctypes.byref(d)) == mpt.LAMP_ERR_INVALID


def test_skip_call_rejects_bad_arguments_on_host():
    L = mpt.lib()
    args = [0x1000] * 7 + [0x2000, 0x3000, 1, 1, 1, 256, 256, 64, 1, 0, 0.0]
    adaptive = mpt.mode_bits("adaptive")
    # bitmask mode, skip below tau, NaN threshold
    assert L.lamp_attn_fwd_q8_skip(*args, mpt.mode_bits("bitmask"), 2.0, 8.0, None, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_attn_fwd_q8_skip(*args, adaptive, 4.0, 2.0, None, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_attn_fwd_q8_skip(*args, adaptive, 4.0, float("nan"), None, None) == mpt.LAMP_ERR_INVALID


def test_decode_rejects_bad_arguments_on_host():
    L = mpt.lib()
    ptrs = [0x1000] * 10  # q, q8, q_scale, k8, k_scale, v8, v_scale, len_k, o, lse
    bitmask = mpt.mode_bits("bitmask")

    def call(p=ptrs, B=1, H=4, Hkv=1, max_k=256, D=128, scale=0.0, mask=None, gt=1, mode=bitmask):
        return L.lamp_decode_fwd(*p, B, H, Hkv, max_k, D, scale, mask, gt, mode, None)

    assert call(p=[None] + ptrs[1:]) == mpt.LAMP_ERR_INVALID              # null query
    assert call(p=ptrs[:3] + [0x1008] + ptrs[4:]) == mpt.LAMP_ERR_INVALID  # k8 not 16-byte aligned
    assert call(mode=mpt.mode_bits("adaptive")) == mpt.LAMP_ERR_UNSUPPORTED
    assert call(mode=mpt.mode_bits(out="in")) == mpt.LAMP_ERR_UNSUPPORTED
    assert call(H=16, Hkv=1) == mpt.LAMP_ERR_UNSUPPORTED                  # 16 query heads per KV head
    assert call(H=3, Hkv=2) == mpt.LAMP_ERR_INVALID
    assert call(max_k=0) == mpt.LAMP_ERR_INVALID
    assert call(D=96) == mpt.LAMP_ERR_UNSUPPORTED
    assert call(scale=float("nan")) == mpt.LAMP_ERR_INVALID
    assert call(mask=0x4000, gt=0) == mpt.LAMP_ERR_INVALID


def test_varlen_calls_reject_bad_arguments_on_host():
    L = mpt.lib()
    m = mpt.mode_bits("bitmask")
    # quantiser: q set without its offsets, a non-positive total, misaligned input
    assert L.lamp_quant_qk_varlen(0x1000, None, 0x2000, None, 0x3000, None, None, None,
                                  1, 2, 1, 256, 256, 256, 256, 128, m, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_quant_qk_varlen(0x1000, None, 0x2000, None, 0x3000, None, 0x4000, None,
                                  1, 2, 1, 256, 256, 0, 256, 128, m, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_quant_qk_varlen(0x1008, None, 0x2000, None, 0x3000, None, 0x4000, None,
                                  1, 2, 1, 256, 256, 256, 256, 128, m, None) == mpt.LAMP_ERR_INVALID
    # attention on precomputed codes: missing offsets
    base = [0x1000] * 9
    assert L.lamp_attn_fwd_q8_varlen(*base, None, 0x5000, 1, 2, 1, 256, 256, 256, 256, 128, 1, 0,
                                     0.0, None, 1, m, 0.0, None, None) == mpt.LAMP_ERR_INVALID
    # full call: null operand, non-positive totals, o not 32-byte aligned, unsupported D
    full = dict(B=1, H=2, Hkv=1, max_q=256, max_k=256, total_q=256, total_k=256, D=128)

    def fwd(q=0x1000, o=0x2000, cu=0x3000, **kw):
        a = {**full, **kw}
        return L.lamp_attn_fwd_varlen(q, 0x1000, 0x1000, o, 0x4000, cu, cu, a["B"], a["H"], a["Hkv"],
                                      a["max_q"], a["max_k"], a["total_q"], a["total_k"], a["D"],
                                      1, 0, 0.0, None, 1, m, 0.0, None)

    assert fwd(q=None) == mpt.LAMP_ERR_INVALID
    assert fwd(cu=None) == mpt.LAMP_ERR_INVALID
    assert fwd(total_q=0) == mpt.LAMP_ERR_INVALID
    assert fwd(o=0x2010) == mpt.LAMP_ERR_INVALID
    assert fwd(D=80) == mpt.LAMP_ERR_UNSUPPORTED


def test_debug_and_exp2_entries_reject_bad_arguments_on_host():
    L = mpt.lib()
    base = [0x1000] * 9 + [1, 1, 1, 128, 128, 128, 1, 0, 0.0, None, 1, 0, 0.0, None]
    # no slot map, n_slots < 1, no dump buffer, misaligned dump buffer
    assert L.lamp_attn_debug(*base, None, 1, 0x2000, None, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_attn_debug(*base, 0x3000, 0, 0x2000, None, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_attn_debug(*base, 0x3000, 1, None, None, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_attn_debug(*base, 0x3000, 1, 0x2004, None, None) == mpt.LAMP_ERR_INVALID
    # the attention checks apply too (window without causal)
    bad = list(base)
    bad[15], bad[16] = 0, 16
    assert L.lamp_attn_debug(*bad, 0x3000, 1, 0x2000, None, None) == mpt.LAMP_ERR_UNSUPPORTED
    assert L.lamp_exp2_eval(None, 0x1000, 4, 0, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_exp2_eval(0x1000, 0x1000, 4, 2, None) == mpt.LAMP_ERR_INVALID
    assert L.lamp_exp2_eval(0x1000, 0x1000, -1, 0, None) == mpt.LAMP_ERR_INVALID
