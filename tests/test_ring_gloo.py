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

    def _scores(self, q, k, causal, scale, q_seg, k_seg):
        s = torch.einsum("bshd,bthd->bhst", q, k) * scale
        n = q.shape[1]
        masked = torch.zeros(q.shape[0], 1, n, n, dtype=torch.bool)
        if causal:
            masked |= torch.ones(n, n, dtype=torch.bool).triu(1)
        if q_seg is not None:
            masked |= (q_seg[:, None, :, None] != k_seg[:, None, None, :]) | (q_seg[:, None, :, None] < 0)
        return s.masked_fill(masked, float("-inf"))

    def block_fwd(self, q, k, v, causal, scale, q_seg=None, k_seg=None):
        scale = scale or 1.0 / np.sqrt(q.shape[-1])
        s = self._scores(q, k, causal, scale, q_seg, k_seg)
        lse = torch.logsumexp(s, -1)
        w = torch.where(torch.isinf(lse)[..., None], torch.zeros_like(s), torch.exp(s - lse[..., None]))
        o = torch.einsum("bhst,bthd->bshd", w, v)
        return o, lse

    def block_bwd(self, q, k, v, o, lse, d_o, causal, scale, q_seg=None, k_seg=None):
        scale = scale or 1.0 / np.sqrt(q.shape[-1])
        s = self._scores(q, k, causal, scale, q_seg, k_seg)
        p = torch.where(torch.isinf(lse)[..., None], torch.zeros_like(s),
                        torch.exp(s - lse[..., None]))  # global LSE
        dp = torch.einsum("bshd,bthd->bhst", d_o, v)
        dsum = (d_o * o).sum(-1).permute(0, 2, 1)[..., None]
        ds = p * (dp - dsum)
        dq = torch.einsum("bhst,bthd->bshd", ds, k) * scale
        dk = torch.einsum("bhst,bshd->bthd", ds, q) * scale
        dv = torch.einsum("bhst,bshd->bthd", p, d_o)
        return dq, dk, dv

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        new = torch.logaddexp(lse_acc, lse_part)
        fin = torch.isfinite(new)
        wa = torch.where(fin, torch.exp(lse_acc - new), torch.zeros_like(new))
        wp = torch.where(fin, torch.exp(lse_part - new), torch.zeros_like(new))
        o_acc.copy_(wa.permute(0, 2, 1)[..., None] * o_acc + wp.permute(0, 2, 1)[..., None] * o_part)
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


def _segments(S, packed):
    if not packed:
        return None
    rng = np.random.default_rng(S)
    cuts = np.sort(rng.choice(np.arange(1, S), size=4, replace=False))
    seg = np.searchsorted(cuts, np.arange(S), side="right")[None].astype(np.int32)
    seg[0, -2:] = -1  # padding at the end
    return seg


def _worker(rank, size, port, n, theta, layout, packed, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=size,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from long_context_causal_attention_b200 import ring as mod
        q, k, v, do = (mod.split_for_ranks(torch.from_numpy(a), size, layout)[rank]
                       for a in _inputs(size * n))
        seg = _segments(size * n, packed)
        seg = None if seg is None else mod.split_for_ranks(torch.from_numpy(seg), size, layout)[rank]
        ops = CpuBlockOps()
        o, lse = mod.ring_forward(q, k, v, theta, ops=ops, layout=layout, segment_ids=seg)
        dq, dk, dv = mod.ring_backward(q, k, v, o, lse, do, theta, ops=ops, layout=layout,
                                       segment_ids=seg)
        out.put((rank, o.numpy(), lse.numpy(), dq.numpy(), dk.numpy(), dv.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("size,n,layout,packed", [(2, 24, "contiguous", False),
                                                  (3, 16, "contiguous", True),
                                                  (2, 24, "zigzag", True), (3, 18, "zigzag", False)])
def test_ring_on_gloo_ranks_matches_oracle(size, n, layout, packed):
    import oracle
    from long_context_causal_attention_b200 import ring
    theta = 300.0
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, size, port, n, theta, layout, packed, out))
             for r in range(size)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in range(size)), key=lambda t: t[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    q, k, v, do = _inputs(size * n)
    ref = oracle.attention_backward(q, k, v, do, _segments(size * n, packed), causal=True,
                                    theta=theta)
    cat = lambda i, ax: ring.merge_from_ranks([torch.from_numpy(r[i]) for r in res], layout,
                                              dim=ax).numpy()
    np.testing.assert_allclose(cat(1, 1), ref["o"], atol=1e-10)
    lse = cat(2, 2)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref["lse"]))
    fin = np.isfinite(ref["lse"])
    np.testing.assert_allclose(lse[fin], ref["lse"][fin], atol=1e-10)
    np.testing.assert_allclose(cat(3, 1), ref["dq"], atol=1e-10)
    np.testing.assert_allclose(cat(4, 1), ref["dk"], atol=1e-10)
    np.testing.assert_allclose(cat(5, 1), ref["dv"], atol=1e-10)
