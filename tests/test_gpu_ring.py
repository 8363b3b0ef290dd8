"""Ring (sequence-parallel) attention on one GPU: N virtual ranks in lockstep.

The sequence is split into N blocks (contiguous layout) or 2N chunks
(zigzag layout, two per rank); the ring runs the library's block kernels
(rotation at each chunk's offset, lwm_attn_fwd / lwm_attn_bwd on the
rotated blocks, the log-sum-exp merge, fp32 gradient accumulation) exactly
as N ranks would, with the shift between ranks a rotation of a list.  The
result must match the float64 oracle on the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_ranks,n,theta,layout", [(4, 256, 1e6, "zigzag"), (3, 384, 1e7, "contiguous"),
                                                   (2, 200, 1e4, "zigzag"), (4, 128, 1e6, "contiguous"),
                                                   (8, 128, 1e6, "zigzag"), (8, 256, 1e7, "contiguous")])
def test_emulated_ring_matches_oracle(n_ranks, n, theta, layout):
    from long_context_causal_attention_b200 import ring
    B, H, D = 1, 4, 128
    S = n_ranks * n
    g = torch.Generator(device="cuda")
    g.manual_seed(n_ranks * 1000 + n)
    q, k, v = ((torch.randn((B, S, H, D), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
               for _ in range(3))
    do = torch.randn((B, S, H, D), generator=g, device="cuda").to(torch.bfloat16)
    split = lambda t, dim=1: ring.split_for_ranks(t, n_ranks, layout, dim)
    res = ring.emulated_ring_forward(split(q), split(k), split(v), theta, layout=layout)
    o = ring.merge_from_ranks([r[0] for r in res], layout)
    lse = ring.merge_from_ranks([r[1] for r in res], layout, dim=2)
    grads = ring.emulated_ring_backward(split(q), split(k), split(v), [r[0] for r in res],
                                        [r[1] for r in res], split(do), theta, layout=layout)
    torch.cuda.synchronize()
    dq, dk, dv = (ring.merge_from_ranks([gr[i] for gr in grads], layout) for i in range(3))
    ref = oracle.attention_backward(to64(q), to64(k), to64(v), to64(do), None, causal=True,
                                    theta=theta)
    assert_close("o", to64(o), ref["o"], "bf16")
    assert_close("lse", to64(lse), ref["lse"], "bf16")
    assert_close("dq", to64(dq), ref["dq"], "bf16")
    assert_close("dk", to64(dk), ref["dk"], "bf16")
    assert_close("dv", to64(dv), ref["dv"], "bf16")


@pytest.mark.parametrize("n_ranks,n,layout", [(4, 256, "zigzag"), (3, 300, "contiguous")])
def test_emulated_ring_packed_matches_oracle(n_ranks, n, layout):
    """Packed rows with padding: the segment ids travel with the key blocks and
    every block pair is masked query ids against key ids."""
    import numpy as np
    from long_context_causal_attention_b200 import ring
    from workloads import random_segments
    B, H, D, theta = 2, 2, 128, 1e6
    S = n_ranks * n
    g = torch.Generator(device="cuda")
    g.manual_seed(77 + n)
    q, k, v = ((torch.randn((B, S, H, D), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
               for _ in range(3))
    do = torch.randn((B, S, H, D), generator=g, device="cuda").to(torch.bfloat16)
    seg = random_segments(np.random.default_rng(n), B, S, 40, 500, pad_tail=3)
    seg_d = torch.as_tensor(seg, dtype=torch.int32, device="cuda")
    split = lambda t: ring.split_for_ranks(t, n_ranks, layout)
    segs = split(seg_d)
    res = ring.emulated_ring_forward(split(q), split(k), split(v), theta, layout=layout,
                                     seg_blocks=segs)
    o = ring.merge_from_ranks([r[0] for r in res], layout)
    lse = ring.merge_from_ranks([r[1] for r in res], layout, dim=2)
    grads = ring.emulated_ring_backward(split(q), split(k), split(v), [r[0] for r in res],
                                        [r[1] for r in res], split(do), theta, layout=layout,
                                        seg_blocks=segs)
    torch.cuda.synchronize()
    dq, dk, dv = (ring.merge_from_ranks([gr[i] for gr in grads], layout) for i in range(3))
    ref = oracle.attention_backward(to64(q), to64(k), to64(v), to64(do), seg, causal=True,
                                    theta=theta)
    assert_close("o", to64(o), ref["o"], "bf16")
    assert_close("lse", to64(lse), ref["lse"], "bf16")
    assert_close("dq", to64(dq), ref["dq"], "bf16")
    assert_close("dk", to64(dk), ref["dk"], "bf16")
    assert_close("dv", to64(dv), ref["dv"], "bf16")


def test_merge_kernel_equals_joint_softmax():
    """Merging the results of two key halves equals attention over both."""
    import long_context_causal_attention_b200 as lwm
    B, S, H, D = 2, 300, 2, 128
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    q = (torch.randn((B, S, H, D), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    k1, k2, v1, v2 = ((torch.randn((B, S, H, D), generator=g, device="cuda") * 0.5)
                      .to(torch.bfloat16) for _ in range(4))
    o1, l1 = lwm.lwm_attn_fwd(q, k1, v1, None, False, 0.0)
    o2, l2 = lwm.lwm_attn_fwd(q, k2, v2, None, False, 0.0)
    o_acc = torch.zeros((B, S, H, D), dtype=torch.float32, device="cuda")
    l_acc = torch.full((B, H, S), float("-inf"), device="cuda")
    lwm.lwm_attn_merge(o_acc, l_acc, o1, l1)
    lwm.lwm_attn_merge(o_acc, l_acc, o2, l2)
    torch.cuda.synchronize()
    # joint reference: plain softmax attention of q over all 2S keys, float64
    K, V = to64(torch.cat([k1, k2], 1)), to64(torch.cat([v1, v2], 1))
    s = np.einsum("bshd,bthd->bhst", to64(q), K) / np.sqrt(D)
    m = s.max(-1, keepdims=True)
    e = np.exp(s - m)
    ref_l = (m[..., 0] + np.log(e.sum(-1)))
    ref_o = np.einsum("bhst,bthd->bshd", e / e.sum(-1, keepdims=True), V)
    assert_close("o", to64(o_acc), ref_o, "bf16")
    assert_close("lse", to64(l_acc), ref_l, "bf16")


def test_fp32_block_results_are_the_bf16_ones_unrounded():
    """The fp32-output pair calls return what the bf16 pair calls round: each
    bf16 result lies within half a bf16 ulp of the fp32 one (2^-9 relative;
    2^-8 allowed, since dq's fp32 partial sums are added in an order that
    differs between launches), for the forward O and the backward dq, dk,
    dv."""
    import long_context_causal_attention_b200 as lwm
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    B, S, H, D = 1, 300, 2, 128
    q, k, v, do = (torch.randn((B, S, H, D), generator=g, device="cuda").to(torch.bfloat16)
                   for _ in range(4))
    o16, lse16 = lwm.lwm_attn_fwd_pair(q, k, v, None, None, True, 0.0)
    o32, lse32 = lwm.lwm_attn_fwd_pair_f32(q, k, v, None, None, True, 0.0)
    g16 = lwm.lwm_attn_bwd_pair(q, k, v, o16, lse16, do, None, None, True, 0.0)
    g32 = lwm.lwm_attn_bwd_pair_f32(q, k, v, o16, lse16, do, None, None, True, 0.0)
    torch.cuda.synchronize()
    assert o32.dtype == torch.float32 and torch.equal(lse16, lse32)
    for a16, a32 in zip((o16,) + tuple(g16), (o32,) + tuple(g32)):
        assert a32.dtype == torch.float32
        ref = a16.float()
        assert bool(((a32 - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-6).all())
        assert not torch.equal(a32, ref)  # the fp32 results are not rounded
