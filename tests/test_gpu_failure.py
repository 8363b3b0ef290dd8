"""Failure detection without a GPU fault.

Every wait of the tensor-core kernels is bounded: when it runs out, the
kernel raises its abort flag, writes LWM_ERR_TIMEOUT into the workspace
status word and returns, and the context stays usable.  The self-test entry
point runs that same wait on a barrier nothing arrives on (with a limit of a
few milliseconds) and on one that is armed; the test checks the status the
host reads back in both cases, and that an ordinary call still succeeds
afterwards on the same context.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    import long_context_causal_attention_b200 as lwm
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    limit = 4_000_000  # ~2 ms of SM clock
    assert lwm.lwm_attn_selftest_wait(ws, limit, arrive=False) == -6  # LWM_ERR_TIMEOUT
    where = int(ws[4:8].view(torch.int32).item())
    assert where == 99
    assert lwm.lwm_attn_selftest_wait(ws, limit, arrive=True) == 0
    # the context is still healthy: a real call runs and reports no error
    q = torch.randn(1, 300, 2, 128, device="cuda").to(torch.bfloat16)
    o, lse = lwm.lwm_attn_fwd(q, q, q, None, True, 1e4, check_status=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
