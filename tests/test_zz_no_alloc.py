"""lwm_attn_fwd_noalloc: the forward pass for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run attention (a memory
planner that forbids new device allocations after start-up, or code that
must not take the synchronisation or out-of-memory risk of one).  For them
the library keeps a fixed 40 MiB scratch array per device and this entry
point uses it instead of a caller workspace.  The test calls it through the
C ABI twice in a row, on two different inputs, and checks each result
against the ordinary lwm_attn_fwd (own workspace) and against the float64
oracle, within the bf16 parity bound, and reads the device status word of
each call back through lwm_attn_fwd_noalloc_read_status; it also checks that
a problem too big for the array is refused before anything runs.  This file is collected last so that a failure here cannot
stop the other tests from running.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import assert_close, to64
from workloads import Workload, make_tensors, random_segments

pytestmark = pytest.mark.gpu


def _noalloc(lwm, q, k, v, seg, theta):
    lib = lwm._lib.lib()
    desc = lwm.make_desc(q, seg, True, theta, 0.0)
    B, S, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    st = lib.lwm_attn_fwd_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  o.data_ptr(), lse.data_ptr(),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, o, lse


def test_noalloc_forward_matches_workspace_forward():
    import long_context_causal_attention_b200 as lwm
    theta = 1e6
    w = Workload("noalloc", 2, 1000, 4, 128, "bf16", theta)
    rng = np.random.default_rng(5)
    seg = torch.as_tensor(random_segments(rng, w.batch, w.seqlen, 50, 400), dtype=torch.int32,
                          device="cuda")
    for seed in (11, 12):  # two calls in a row, different inputs
        t = make_tensors(w, seed=seed, device="cuda", with_grad_out=False)
        st, o, lse = _noalloc(lwm, t["q"], t["k"], t["v"], seg, theta)
        assert st == 0, lwm.lwm_status_string(st)
        dev_st = lwm._lib.lib().lwm_attn_fwd_noalloc_read_status(
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert dev_st == 0, lwm.lwm_status_string(dev_st)
        ref = oracle.attention_forward(to64(t["q"]), to64(t["k"]), to64(t["v"]),
                                       seg.cpu().numpy(), causal=True, theta=theta)
        assert_close("o vs oracle", to64(o), ref[0], "bf16")
        assert_close("lse vs oracle", to64(lse), ref[1], "bf16")
        o_ref, lse_ref = lwm.lwm_attn_fwd(t["q"], t["k"], t["v"], seg, True, theta,
                                          check_status=True)
        torch.cuda.synchronize()
        assert_close("o", to64(o), to64(o_ref), "bf16")
        assert_close("lse", to64(lse), to64(lse_ref), "bf16")


def test_noalloc_refuses_problems_beyond_its_scratch():
    import long_context_causal_attention_b200 as lwm
    lib = lwm._lib.lib()
    # 8 x 4096 tokens x 32 x 128 needs far more than 40 MiB of rotated q/k
    desc = lwm.LwmAttnDesc(8, 4096, 32, 128, 0, 1, 1e6, 0.0, None)
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = lib.lwm_attn_fwd_noalloc(ctypes.byref(desc), fake, fake, fake, fake, fake, None)
    assert st == -4  # LWM_ERR_WORKSPACE
