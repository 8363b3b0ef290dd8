"""Head-parallel split of one problem over ranks, run as gloo ranks on CPU.

Each rank takes its heads of the whole inputs (the scatter), runs attention
on them -- here the float64 oracle stands in for the single-GPU kernels --
and the outputs are gathered back along the head axis.  The result must be
the oracle on the whole problem, exactly: the (batch, head) units are
independent, so the split adds no arithmetic and the data path has no
exchange step.  Packed rows with padding, world sizes 2 and 4.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from workloads import random_segments
    rng = np.random.default_rng(21)
    B, S, H, D = 2, 150, 8, 16
    seg = random_segments(rng, B, S, 10, 60, pad_tail=3)
    g = torch.Generator().manual_seed(5)
    t = {n: torch.randn(B, S, H, D, generator=g, dtype=torch.float64) for n in ("q", "k", "v", "do")}
    return t, seg, 1e6


def _worker(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from long_context_causal_attention_b200.heads import run_head_parallel
        t, seg, theta = _case()

        def step(q, k, v, do):
            r = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), seg,
                                          causal=True, theta=theta)
            return {key: torch.from_numpy(np.ascontiguousarray(r[key]))
                    for key in ("o", "lse", "dq", "dk", "dv")}

        got = run_head_parallel(step, t, rank, ws)
        if rank == 0:
            out.put({key: val.numpy() for key, val in got.items()})
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 4])
def test_head_split_gathers_to_the_whole_problem(ws):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, out)) for r in range(ws)]
    for p in procs:
        p.start()
    got = out.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    t, seg, theta = _case()
    ref = oracle.attention_backward(*(t[n].numpy() for n in ("q", "k", "v", "do")), seg,
                                    causal=True, theta=theta)
    for key in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(np.isfinite(got[key]), np.isfinite(ref[key]))
        fin = np.isfinite(ref[key])
        np.testing.assert_allclose(got[key][fin], ref[key][fin], rtol=0, atol=1e-12)


def test_head_range_splits_evenly_and_refuses_the_rest():
    from long_context_causal_attention_b200.heads import head_range, scatter_heads
    assert [head_range(32, r, 8) for r in range(8)] == [(4 * r, 4 * r + 4) for r in range(8)]
    assert head_range(32, 0, 1) == (0, 32)
    with pytest.raises(ValueError):
        head_range(32, 0, 3)
    with pytest.raises(ValueError):
        head_range(32, 2, 2)
    x = torch.arange(2 * 3 * 4 * 5).reshape(2, 3, 4, 5)
    part = scatter_heads(x, 1, 2)
    assert part.is_contiguous() and torch.equal(part, x[:, :, 2:4])
    lse = torch.arange(2 * 4 * 3).reshape(2, 4, 3)
    assert torch.equal(scatter_heads(lse, 1, 2, head_dim_axis=1), lse[:, 2:4])


def test_bench_counts_the_whole_problem_once_under_a_head_split():
    """Whole-job throughput of a head split: each rank's work is 1/N of the
    problem, and job_tflops(local work, N, slowest time) is the whole
    problem's work over the slowest rank's time."""
    sys.path.insert(0, ROOT)
    import bench
    whole = 3.5 * 4.0 * 128 * 32 * (131072 * 131073 // 2)
    for n in (1, 2, 4, 8):
        local = 3.5 * 4.0 * 128 * (32 // n) * (131072 * 131073 // 2)
        assert bench.job_tflops(local, n, 100.0) == pytest.approx(whole / 0.1 / 1e12)
