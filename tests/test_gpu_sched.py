"""Work distribution of the persistent two-tile attention kernel (GPU).

When its KV planes exceed L2 (more than 100 MB of K16, V and K8 together), the kernel's CTAs
take their work items (query-tile pairs) from a launch-wide ticket counter held in one of the
library's scheduler slots, in an order that takes the KV planes in L2-sized chunks; the CTA
that takes the last ticket returns the slot to idle.  Smaller problems walk a fixed order.
Every item is computed by exactly one CTA whatever the order, and an item's arithmetic does
not depend on the other items of the launch, so the outputs must be bit-identical:
  * to launches on slices of the heads (small enough for the fixed order): every item of the
    large launch was computed, once, exactly as the fixed order computes it;
  * across more launches than there are slots (every slot is reused, so each must have been
    returned to idle);
  * with two launches in flight at once on two streams;
  * across replays of a captured CUDA graph (the same slot and tag every replay);
  * after a forced device-side timeout (lamp_check returns the slots to idle).
"""
import pytest
import torch

import mixed_precision_tiled_b200 as mpt

pytestmark = pytest.mark.gpu

D = 128
# 8 KV planes of 19600 keys: 8 * 5 * 19600 * 128 bytes = 100.4 MB > 100 MB (ticket counter)
L_BIG = 19600


def _case(B, H, Hkv, L, seed, g=2, p16=0.3, route="bitmask", dt=torch.bfloat16):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((B, H, L, D), generator=gen).to(dt).cuda()
    k = torch.randn((B, Hkv, L, D), generator=gen).to(dt).cuda()
    v = torch.randn((B, Hkv, L, D), generator=gen).to(dt).cuda()
    q8, k8, qs, ks = mpt.quantize(q, k)
    if route == "adaptive":
        return [q, k, v, q8, k8, qs, ks], dict(causal=True, route="adaptive", tau=4.0)
    mask = mpt.build_mask(B, H, L, L, D, g, p16, seed)
    return [q, k, v, q8, k8, qs, ks], dict(causal=True, mask_bits=mask, group_tiles=g)


def _run(args, kw, stream=None):
    return mpt.attention_q8(*args, **kw, stream=stream)


def _head_slice(args, kw, h0, h1, kv0, kv1):
    q, k, v, q8, k8, qs, ks = args
    sub = [q[:, h0:h1], k[:, kv0:kv1], v[:, kv0:kv1], q8[:, h0:h1], k8[:, kv0:kv1],
           qs[:, h0:h1], ks[:, kv0:kv1]]
    kw2 = dict(kw, mask_bits=kw["mask_bits"][:, h0:h1]) if "mask_bits" in kw else dict(kw)
    return [x.contiguous() for x in sub], kw2


@pytest.mark.parametrize("H,Hkv,route,dt", [(16, 8, "bitmask", torch.bfloat16),
                                            (8, 8, "bitmask", torch.bfloat16),
                                            (16, 8, "adaptive", torch.bfloat16),
                                            (16, 8, "bitmask", torch.float16)])
def test_ticket_order_equals_fixed_order_on_head_slices(H, Hkv, route, dt):
    # (16, 8): items are one query tile of two heads; (8, 8): two query tiles of one head; the
    # look-ahead and fp16 instantiations of the ticket order too
    args, kw = _case(1, H, Hkv, L_BIG, 11, route=route, dt=dt)
    o, lse = _run(args, kw)
    torch.cuda.synchronize()
    mpt.lamp_check()
    G = H // Hkv
    for kv in range(Hkv):
        sa, skw = _head_slice(args, kw, kv * G, (kv + 1) * G, kv, kv + 1)
        o1, l1 = _run(sa, skw)
        torch.cuda.synchronize()
        assert torch.equal(o[:, kv * G:(kv + 1) * G], o1), kv
        assert torch.equal(lse[:, kv * G:(kv + 1) * G], l1), kv
    mpt.lamp_check()


def test_more_launches_than_slots():
    args, kw = _case(1, 16, 8, L_BIG, 1)
    o0, lse0 = _run(args, kw)
    torch.cuda.synchronize()
    mpt.lamp_check()
    n = 1100  # > the 1024 scheduler slots: every slot is taken at least once more
    for i in range(n):
        o, lse = _run(args, kw)
        if i % 97 == 0 or i == n - 1:
            torch.cuda.synchronize()
            assert torch.equal(o, o0) and torch.equal(lse, lse0), i
    mpt.lamp_check()


def test_two_streams_in_flight():
    a_args, a_kw = _case(1, 16, 8, L_BIG, 2)
    b_args, b_kw = _case(1, 8, 8, L_BIG, 3)
    oa0, la0 = _run(a_args, a_kw)
    ob0, lb0 = _run(b_args, b_kw)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        outs.append(_run(a_args, a_kw, s1) + _run(b_args, b_kw, s2))
    torch.cuda.synchronize()
    mpt.lamp_check()
    for oa, la, ob, lb in outs:
        assert torch.equal(oa, oa0) and torch.equal(la, la0)
        assert torch.equal(ob, ob0) and torch.equal(lb, lb0)


def test_graph_replays():
    args, kw = _case(1, 16, 8, L_BIG, 4)
    o0, lse0 = _run(args, kw)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        _run(args, kw)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        o, lse = _run(args, kw)
    for _ in range(4):
        o.zero_()
        lse.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o0) and torch.equal(lse, lse0)
    mpt.lamp_check()
    del graph


def test_launch_after_forced_timeout():
    args, kw = _case(1, 16, 8, L_BIG, 5)
    o0, lse0 = _run(args, kw)
    torch.cuda.synchronize()
    mpt.lamp_selftest_timeout(1_000_000)  # 1 ms on a barrier nothing completes
    with pytest.raises(mpt.LampError) as e:
        mpt.lamp_check()
    assert e.value.code == mpt.LAMP_ERR_TIMEOUT
    for _ in range(3):
        o, lse = _run(args, kw)
        torch.cuda.synchronize()
        assert torch.equal(o, o0) and torch.equal(lse, lse0)
    mpt.lamp_check()
