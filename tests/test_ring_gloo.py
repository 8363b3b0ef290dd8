"""Ring attention's exchange schedule on world-size 2 and 3 gloo ranks (CPU).

The ring stepping loop for torch.distributed (NCCL on GPUs) runs here on gloo
ranks with a CPU stand-in for the block operations (float64 torch math, the
oracle's rotation), so the point-to-point schedule, the causal skipping of
later blocks, the log-sum-exp merge order and the final shift that brings
dk/dv home are checked against the oracle on the whole sequence without a
GPU.  The GPU path runs the same per-rank algorithm with the library's
kernels (tests/test_gpu_ring.py).
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


class CpuBlockOps:
    """float64 CPU versions of the ring's block operations (test only)."""

    def rotate(self, x, theta, pos0, inverse=False):
        import oracle
        y = oracle.rope_apply(x.numpy(), theta, inverse=inverse, position_offset=pos0)
        return torch.from_numpy(y)

    def _scores(self, q, k, causal, scale):
        s = torch.einsum("bshd,bthd->bhst", q, k) * scale
        if causal:
            n = q.shape[1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        return s

    def block_fwd(self, q, k, v, causal, scale):
        scale = scale or 1.0 / np.sqrt(q.shape[-1])
        s = self._scores(q, k, causal, scale)
        lse = torch.logsumexp(s, -1)
        o = torch.einsum("bhst,bthd->bshd", torch.exp(s - lse[..., None]), v)
        return o, lse

    def block_bwd(self, q, k, v, o, lse, d_o, causal, scale):
        scale = scale or 1.0 / np.sqrt(q.shape[-1])
        p = torch.exp(self._scores(q, k, causal, scale) - lse[..., None])  # global LSE
        dp = torch.einsum("bshd,bthd->bhst", d_o, v)
        dsum = (d_o * o).sum(-1).permute(0, 2, 1)[..., None]
        ds = p * (dp - dsum)
        dq = torch.einsum("bhst,bthd->bshd", ds, k) * scale
        dk = torch.einsum("bhst,bshd->bthd", ds, q) * scale
        dv = torch.einsum("bhst,bshd->bthd", p, d_o)
        return dq, dk, dv

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        m = torch.maximum(lse_acc, lse_part)
        new = m + torch.log(torch.exp(lse_acc - m) + torch.exp(lse_part - m))
        wa = torch.exp(lse_acc - new).permute(0, 2, 1)[..., None]
        wp = torch.exp(lse_part - new).permute(0, 2, 1)[..., None]
        o_acc.copy_(wa * o_acc + wp * o_part)
        lse_acc.copy_(new)

    def accumulate(self, acc, x):
        acc += x

    def convert(self, x, dtype):
        return x.clone()

    def zeros_f32(self, shape, device):
        return torch.zeros(shape, dtype=torch.float64)

    def full_f32(self, shape, value, device):
        return torch.full(shape, value, dtype=torch.float64)


def _inputs(S, seed=7):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((1, S, 2, 8)) for _ in range(4)]  # q, k, v, dO


def _worker(rank, size, port, n, theta, layout, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=size,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from long_context_causal_attention_b200 import ring as mod
        q, k, v, do = (mod.split_for_ranks(torch.from_numpy(a), size, layout)[rank]
                       for a in _inputs(size * n))
        ops = CpuBlockOps()
        o, lse = mod.ring_forward(q, k, v, theta, ops=ops, layout=layout)
        dq, dk, dv = mod.ring_backward(q, k, v, o, lse, do, theta, ops=ops, layout=layout)
        out.put((rank, o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("size,n,layout", [(2, 24, "contiguous"), (3, 16, "contiguous"),
                                           (2, 24, "zigzag"), (3, 18, "zigzag")])
def test_ring_on_gloo_ranks_matches_oracle(size, n, layout):
    import oracle
    from long_context_causal_attention_b200 import ring
    theta = 300.0
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, size, port, n, theta, layout, out))
             for r in range(size)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in range(size)), key=lambda t: t[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    q, k, v, do = _inputs(size * n)
    ref = oracle.attention_backward(q, k, v, do, None, causal=True, theta=theta)
    cat = lambda i, ax: ring.merge_from_ranks([torch.from_numpy(r[i]) for r in res], layout,
                                              dim=ax).numpy()
    np.testing.assert_allclose(cat(1, 1), ref["o"], atol=1e-10)
    np.testing.assert_allclose(cat(2, 2), ref["lse"], atol=1e-10)
    np.testing.assert_allclose(cat(3, 1), ref["dq"], atol=1e-10)
    np.testing.assert_allclose(cat(4, 1), ref["dk"], atol=1e-10)
    np.testing.assert_allclose(cat(5, 1), ref["dv"], atol=1e-10)
