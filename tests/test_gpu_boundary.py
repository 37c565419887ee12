"""The boundary's error contract on a real device (GPU): a rejected call enqueues nothing.

The end-to-end entry points (lamp_attn_fwd, lamp_attn_fwd_noalloc, lamp_attn_fwd_varlen)
quantise into a workspace and then run the attention kernel.  Every argument check must come
before either step: a call that returns an error code has launched no kernel, written no
workspace byte and left o / lse as they were.  Two independent witnesses:
  * sentinel-filled o, lse and a caller-set workspace stay bit-identical after the call;
  * the call made inside a stream capture adds no node to the captured graph.
"""
import math

import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt

pytestmark = pytest.mark.gpu

B, H, Hkv, L, D = 1, 4, 2, 300, 128
SENT = 12345.0


def _inputs():
    g = torch.Generator(device="cpu").manual_seed(7)
    q = torch.randn((B, H, L, D), generator=g).to(torch.bfloat16).cuda()
    k = torch.randn((B, Hkv, L, D), generator=g).to(torch.bfloat16).cuda()
    v = torch.randn((B, Hkv, L, D), generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def _outputs():
    # one spare element so that a misaligned o can be made from the same buffer
    o_buf = torch.full((B * H * L * D + 8,), SENT, device="cuda", dtype=torch.float32)
    lse = torch.full((B, H, L), SENT, device="cuda", dtype=torch.float32)
    return o_buf, lse


BAD = [
    ("window without causal", dict(causal=0, window=64), mpt.LAMP_ERR_UNSUPPORTED),
    ("unknown mode bits", dict(mode=0x30), mpt.LAMP_ERR_INVALID),
    ("group_tiles 0", dict(group_tiles=0), mpt.LAMP_ERR_INVALID),
    ("NaN tau", dict(mode=mpt.mode_bits("adaptive"), tau=math.nan), mpt.LAMP_ERR_INVALID),
    ("NaN scale", dict(scale=math.nan), mpt.LAMP_ERR_INVALID),
    ("o not 32-byte aligned", dict(o_off=1), mpt.LAMP_ERR_INVALID),
    ("negative window", dict(window=-2), mpt.LAMP_ERR_INVALID),
    ("causal 2", dict(causal=2), mpt.LAMP_ERR_INVALID),
]


def _call(entry, q, k, v, o_buf, lse, cu, stream, causal=1, window=0, scale=0.0, mode=None,
          tau=0.0, group_tiles=1, o_off=0):
    mode = mpt.mode_bits("bitmask") if mode is None else mode
    o = o_buf.data_ptr() + 4 * o_off
    L_ = mpt.lib()
    s = stream.cuda_stream
    if entry == "fwd":
        return L_.lamp_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o, lse.data_ptr(), B, H,
                                Hkv, L, L, D, causal, window, scale, None, group_tiles, mode,
                                tau, s)
    if entry == "noalloc":
        return L_.lamp_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o,
                                        lse.data_ptr(), B, H, Hkv, L, L, D, causal, window,
                                        scale, None, group_tiles, mode, tau, s)
    # variable-length batch of one sequence: [H][L][D] packed is the same memory as [1][H][L][D]
    return L_.lamp_attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o, lse.data_ptr(),
                                   cu.data_ptr(), cu.data_ptr(), B, H, Hkv, L, L, L, L, D, causal,
                                   window, scale, None, group_tiles, mode, tau, s)


def _graph_nodes_of(fn, stream):
    """Number of nodes a stream capture records around fn() (relaxed mode: the library's
    non-stream calls such as cudaGetDevice are allowed)."""
    from cuda.bindings import runtime as rt
    h = stream.cuda_stream
    err, = rt.cudaStreamBeginCapture(h, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == rt.cudaError_t.cudaSuccess, err
    try:
        rc = fn()
    finally:
        err, graph = rt.cudaStreamEndCapture(h)
    assert err == rt.cudaError_t.cudaSuccess, err
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    rt.cudaGraphDestroy(graph)
    return rc, int(n)


@pytest.mark.parametrize("entry", ["fwd", "noalloc", "varlen"])
@pytest.mark.parametrize("what,bad,code", BAD, ids=[b[0] for b in BAD])
def test_rejected_call_enqueues_nothing(entry, what, bad, code):
    q, k, v = _inputs()
    o_buf, lse = _outputs()
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    # a caller-owned workspace filled with a sentinel byte: the quantiser would write into it
    need = mpt.lamp_workspace_size(B, H, Hkv, L, L, D)
    ws = torch.full((need + 256,), 0xAB, dtype=torch.uint8, device="cuda")
    ws_ptr = (ws.data_ptr() + 255) & ~255
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    try:
        if entry != "noalloc":
            mpt.lamp_set_workspace(ws_ptr, need)
        rc = _call(entry, q, k, v, o_buf, lse, cu, stream, **bad)
        assert rc == code, (what, rc, mpt.lamp_last_error())
        torch.cuda.synchronize()
        assert torch.all(o_buf == SENT) and torch.all(lse == SENT), what
        assert torch.all(ws == 0xAB), f"{what}: the workspace was written"
        rc, nodes = _graph_nodes_of(lambda: _call(entry, q, k, v, o_buf, lse, cu, stream, **bad),
                                    stream)
        assert rc == code and nodes == 0, (what, rc, nodes)
    finally:
        mpt.lamp_set_workspace(None, 0)
    mpt.lamp_check(stream)


@pytest.mark.parametrize("entry", ["fwd", "noalloc", "varlen"])
def test_valid_call_still_runs(entry):
    # the same buffers with valid arguments: o and lse are written, and all three entry points
    # agree bit for bit (one launch configuration, one quantiser)
    q, k, v = _inputs()
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    o_buf, lse = _outputs()
    torch.cuda.synchronize()  # inputs were made on the default stream
    assert _call(entry, q, k, v, o_buf, lse, cu, stream) == mpt.LAMP_OK, mpt.lamp_last_error()
    mpt.lamp_check(stream)
    o = o_buf[:B * H * L * D]
    assert torch.isfinite(o).all() and not torch.any(lse == SENT)
    ref_o, ref_lse = _outputs()
    torch.cuda.synchronize()
    assert _call("fwd", q, k, v, ref_o, ref_lse, cu, stream) == mpt.LAMP_OK
    mpt.lamp_check(stream)
    assert torch.equal(o, ref_o[:B * H * L * D]) and torch.equal(lse, ref_lse)


def test_workspace_grows_in_stream_order():
    # the cached workspace is grown by a larger call on a side stream right after a smaller
    # one; both results match the 8-bit-operand path on the same inputs
    stream = torch.cuda.Stream()
    outs = []
    for Lx in (256, 2048):
        g = torch.Generator(device="cpu").manual_seed(Lx)
        q = torch.randn((1, 2, Lx, D), generator=g).to(torch.bfloat16).cuda()
        k = torch.randn((1, 1, Lx, D), generator=g).to(torch.bfloat16).cuda()
        v = torch.randn((1, 1, Lx, D), generator=g).to(torch.bfloat16).cuda()
        stream.wait_stream(torch.cuda.current_stream())
        o, lse = mpt.attention(q, k, v, causal=True, stream=stream)
        q8, k8, qs, ks = mpt.quantize(q, k, stream=stream)
        o2, lse2 = mpt.attention_q8(q, k, v, q8, k8, qs, ks, causal=True, stream=stream)
        outs.append((o, lse, o2, lse2))
    mpt.lamp_check(stream)
    for o, lse, o2, lse2 in outs:
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
