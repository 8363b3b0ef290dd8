"""Host logic of the multi-GPU benchmark, run as world-size-2 gloo ranks on CPU.

Each GPU runs an independent problem (different seed, same shape), so the
data path has no collective; the only cross-rank steps are the barrier and the
max-over-ranks reduction of the timings, and the whole-job throughput counts
the work of every rank over the slowest rank's time.  These tests run those
helpers of bench.py on two gloo ranks, and check that a rank that dies before
the reduction makes the survivor fail with an error instead of waiting.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, ws, port, seconds=30):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=seconds))


def _reduce_worker(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from workloads import WORKLOADS, make_tensors
    _init(rank, ws, port)
    try:
        assert bench.dist_setup() == (ws, rank, rank)
        # rank r took (10 + r) ms per step on its own problem
        ms, other = bench.max_over_ranks([10.0 + rank, 5.0 - rank], ws, "cpu")
        w = WORKLOADS["tiny_packed_fp32"]
        t = make_tensors(w, seed=bench.rank_seed(0, rank), device="cpu")
        gathered = [torch.empty_like(t["q"]) for _ in range(ws)]
        dist.all_gather(gathered, t["q"])
        out.put((rank, ms, other, bench.job_tflops(2e12, ws, ms),
                 bool(torch.equal(gathered[0], gathered[1])), tuple(t["q"].shape)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reduce_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    for rank, ms, other, tflops, same, shape in res:
        assert ms == 11.0 and other == 5.0          # both ranks see the maxima
        assert tflops == pytest.approx(2 * 2e12 / 11e-3 / 1e12)  # all work / slowest time
        assert not same                                # independent problems per rank
        assert shape == (1, 256, 1, 64)                # of the same shape


def _dying_worker(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, ws, port, seconds=5)
    if rank == 1:
        os._exit(3)  # this rank dies between steps, before the timing reduction
    try:
        bench.max_over_ranks([1.0], ws, "cpu")
        out.put("returned")
    except Exception as e:  # noqa: BLE001 - any error is the expected outcome
        out.put("error: " + type(e).__name__)


def test_dead_rank_ends_the_reduction_with_an_error():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    msg = out.get(timeout=5)
    assert msg.startswith("error"), msg


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(workload="long_128k", seed=0, oracle_rows=8, warmup=0, steps=1))
    assert bench.reference_arm(args) == 0
    assert capsys.readouterr().out == ""
