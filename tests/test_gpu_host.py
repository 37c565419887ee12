"""lamp_attn_fwd_host: the end-to-end call on host buffers (GPU).

The call cuts the B * Hkv KV planes into chunks and pipelines host-to-device copies, the
quantiser and the attention kernel, and device-to-host copies through two device slots.  Each
KV plane (one KV head with its query heads) is an independent problem, so the host results
must be bit-identical to lamp_attn_fwd on the same inputs in device memory, for every chunking
(one chunk, ragged chunks, one plane per chunk), with pinned or pageable host buffers, with
and without lse, and with O in fp32 or in the input dtype.
"""
import math

import pytest
import torch

import mixed_precision_tiled_b200 as mpt

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, Hkv, L, D, window, route, fmt, n_chunks
    (2, 8, 4, 1000, 128, 0, "bitmask", "int8", 3),      # 8 planes: chunks of 3, 3, 2
    (2, 8, 4, 1000, 128, 0, "bitmask", "int8", 0),      # automatic: one chunk
    (1, 4, 4, 700, 64, 0, "bitmask", "int8", 4),        # one plane per chunk, odd group
    (1, 8, 4, 900, 256, 256, "bitmask", "int8", 2),     # D = 256, sliding window
    (3, 4, 2, 600, 128, 0, "adaptive", "e4m3", 5),      # look-ahead, E4M3, 6 planes
]


def _device_inputs(B, H, Hkv, L, D, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, H, L, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, L, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, D), generator=g).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("B,H,Hkv,L,D,window,route,fmt,n_chunks", CASES)
@pytest.mark.parametrize("pinned", [True, False])
def test_host_call_equals_device_call(B, H, Hkv, L, D, window, route, fmt, n_chunks, pinned):
    q, k, v = _device_inputs(B, H, Hkv, L, D, seed=B * 100 + D + n_chunks)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    mode = mpt.mode_bits(route, fmt, "bf16")
    g = 2
    mask = mpt.build_mask(B, H, L, L, D, g, 0.3, 5) if route == "bitmask" else None
    tau = 4.0 if route == "adaptive" else 0.0
    o_ref = torch.empty((B, H, L, D), device="cuda", dtype=torch.float32)
    l_ref = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
    mpt.lamp_attn_fwd(dq, dk, dv, o_ref, l_ref, B, H, Hkv, L, L, D, 1, window, 0.0, mask, g, mode,
                      tau)
    hq, hk, hv = (x.pin_memory() if pinned else x.clone() for x in (q, k, v))
    ho = torch.full((B, H, L, D), math.nan, dtype=torch.float32)
    hl = torch.full((B, H, L), math.nan, dtype=torch.float32)
    if pinned:
        ho, hl = ho.pin_memory(), hl.pin_memory()
    mpt.lamp_attn_fwd_host(hq, hk, hv, ho, hl, B, H, Hkv, L, L, D, 1, window, 0.0, mask, g, mode,
                           tau, n_chunks=n_chunks)
    torch.cuda.synchronize()
    mpt.lamp_check()
    assert torch.equal(ho, o_ref.cpu()) and torch.equal(hl, l_ref.cpu())


def test_host_call_input_dtype_output_and_no_lse():
    B, H, Hkv, L, D = 1, 8, 2, 1500, 128
    q, k, v = _device_inputs(B, H, Hkv, L, D, seed=9)
    mode = mpt.mode_bits("bitmask", "int8", "bf16", "in")
    mask = mpt.build_mask(B, H, L, L, D, 4, 0.25, 3)
    o_ref = torch.empty((B, H, L, D), device="cuda", dtype=torch.bfloat16)
    mpt.lamp_attn_fwd(q.cuda(), k.cuda(), v.cuda(), o_ref, None, B, H, Hkv, L, L, D, 1, 0, 0.0,
                      mask, 4, mode, 0.0)
    ho = torch.zeros((B, H, L, D), dtype=torch.bfloat16).pin_memory()
    hin = [x.pin_memory() for x in (q, k, v)]
    mpt.lamp_attn_fwd_host(*hin, ho, None, B, H, Hkv, L, L, D, 1, 0, 0.0, mask, 4, mode, 0.0,
                           n_chunks=2)
    torch.cuda.synchronize()
    mpt.lamp_check()
    assert torch.equal(ho, o_ref.cpu())


def test_host_calls_back_to_back_on_a_side_stream():
    # consecutive calls reuse the two slots and the copy streams; each must see its own inputs.
    # The references run first: calls on different streams that share the workspace need the
    # caller's ordering.
    B, H, Hkv, L, D = 2, 4, 2, 800, 128
    mode = mpt.mode_bits("bitmask", "int8", "bf16")
    mask = mpt.build_mask(B, H, L, L, D, 1, 0.2, 1)
    inputs, refs = [], []
    for seed in range(3):
        q, k, v = _device_inputs(B, H, Hkv, L, D, seed=seed)
        o_ref = torch.empty((B, H, L, D), device="cuda", dtype=torch.float32)
        mpt.lamp_attn_fwd(q.cuda(), k.cuda(), v.cuda(), o_ref, None, B, H, Hkv, L, L, D, 1, 0,
                          0.0, mask, 1, mode, 0.0)
        inputs.append([x.pin_memory() for x in (q, k, v)])  # alive until the copies are done
        refs.append(o_ref.cpu())
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    outs = []
    for hin in inputs:
        ho = torch.empty((B, H, L, D), dtype=torch.float32).pin_memory()
        mpt.lamp_attn_fwd_host(*hin, ho, None, B, H, Hkv, L, L, D, 1, 0, 0.0, mask, 1, mode, 0.0,
                               n_chunks=4, stream=stream)
        outs.append(ho)
    stream.synchronize()
    mpt.lamp_check(stream)
    for ho, o_ref in zip(outs, refs):
        assert torch.equal(ho, o_ref)
