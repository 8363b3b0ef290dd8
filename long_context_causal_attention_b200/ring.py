"""Sequence-parallel (ring) attention over the library's block kernels.

Blockwise RingAttention, the design the LWM pages train with (research note,
sections "模型架构" and "Infra"; paper card, Summary): the sequence of each
row is split into N equal blocks, block r held by rank r of a ring.  Every
rank keeps its query block and passes its key/value block to the next rank N
times over, so each query block meets every key/value block once; the
per-block results combine exactly by their log-sum-exp, so the result equals
attention over the whole sequence.  With a causal mask, block pairs whose
keys all come after the queries (source rank > own rank) are skipped, the
diagonal pair is causal inside and earlier blocks are attended in full.

Backward: every rank computes, for each visiting key/value block, the
contributions to its own dq and to the visitor's dk and dv (FlashAttention
recomputation with the GLOBAL log-sum-exp and D = dO . O, so block
contributions simply add); the visitor's dk/dv accumulators travel with it
and are home after N shifts.

Each step of the arithmetic runs in the library's CUDA kernels
(lwm_rope_apply_at, lwm_attn_fwd / lwm_attn_bwd on rotated inputs,
lwm_attn_merge, lwm_accumulate, lwm_convert_f32); this module only orders
them and moves blocks.  Two stepping loops run the same per-rank algorithm:
``ring_forward`` / ``ring_backward`` for one rank of a torch.distributed
process group (NCCL point-to-point over NVLink; block i+1 is in flight while
block i is computed), and ``emulated_ring_forward`` / ``..._backward`` for
N virtual ranks stepped in lockstep on one device (same kernels, the shift
is a rotation of a list).  Segment ids (packing) are not supported across
blocks yet.
"""
from __future__ import annotations

import torch

from . import _lib as L


class GpuBlockOps:
    """Per-block operations of the ring, on the library's kernels."""

    def rotate(self, x, theta, pos0, inverse=False):
        return L.lwm_rope_apply_at(x, theta, pos0, inverse)

    def block_fwd(self, q, k, v, causal, scale):
        # inputs are rotated already: rope_theta = 0
        return L.lwm_attn_fwd(q, k, v, None, causal, 0.0, scale)

    def block_bwd(self, q, k, v, o, lse, d_o, causal, scale):
        return L.lwm_attn_bwd(q, k, v, o, lse, d_o, None, causal, 0.0, scale)

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        L.lwm_attn_merge(o_acc, lse_acc, o_part, lse_part)

    def accumulate(self, acc, x):
        L.lwm_accumulate(acc, x)

    def convert(self, x, dtype):
        return L.lwm_convert_f32(x, dtype)

    def zeros_f32(self, shape, device):
        return torch.zeros(shape, dtype=torch.float32, device=device)

    def full_f32(self, shape, value, device):
        return torch.full(shape, value, dtype=torch.float32, device=device)


# ----------------------------------------------------------------------------
# the per-rank algorithm, as generators: ("start", tensors) hands the
# stepping loop the tensors to pass on to the next rank and gets back a
# handle; ("wait", handle) returns the tensors received from the previous rank.
# ----------------------------------------------------------------------------
def _forward_steps(rank, size, q, k, v, theta, scale, ops):
    B, n, H, D = q.shape
    pos0 = rank * n
    qr = ops.rotate(q, theta, pos0)
    blk = [ops.rotate(k, theta, pos0), v]
    o_acc = ops.zeros_f32((B, n, H, D), q.device)
    lse_acc = ops.full_f32((B, H, n), float("-inf"), q.device)
    for s in range(size):
        src = (rank - s) % size
        h = (yield ("start", blk)) if s < size - 1 else None
        if src <= rank:
            o_p, lse_p = ops.block_fwd(qr, blk[0], blk[1], src == rank, scale)
            ops.merge(o_acc, lse_acc, o_p, lse_p)
        if s < size - 1:
            blk = yield ("wait", h)
    return ops.convert(o_acc, q.dtype), lse_acc


def _backward_steps(rank, size, q, k, v, o, lse, d_o, theta, scale, ops):
    B, n, H, D = q.shape
    pos0 = rank * n
    qr = ops.rotate(q, theta, pos0)
    dq_acc = ops.zeros_f32((B, n, H, D), q.device)
    # the visiting block: rotated keys, values and their gradient accumulators
    blk = [ops.rotate(k, theta, pos0), v, ops.zeros_f32((B, n, H, D), q.device),
           ops.zeros_f32((B, n, H, D), q.device)]
    for s in range(size):
        src = (rank - s) % size
        if src <= rank:
            dq_p, dk_p, dv_p = ops.block_bwd(qr, blk[0], blk[1], o, lse, d_o, src == rank, scale)
            ops.accumulate(dq_acc, dq_p)
            ops.accumulate(blk[2], dk_p)
            ops.accumulate(blk[3], dv_p)
        # N shifts in all: after the last one every block is home with its sums
        h = yield ("start", blk)
        blk = yield ("wait", h)
    dq = ops.convert(ops.rotate(dq_acc, theta, pos0, inverse=True), q.dtype)
    dk = ops.convert(ops.rotate(blk[2], theta, pos0, inverse=True), k.dtype)
    dv = ops.convert(blk[3], v.dtype)
    return dq, dk, dv


# ----------------------------------------------------------------------------
# stepping loops
# ----------------------------------------------------------------------------
def _run_distributed(gen, group):
    import torch.distributed as dist
    rank = dist.get_rank(group)
    size = dist.get_world_size(group)
    nxt = dist.get_global_rank(group, (rank + 1) % size) if group is not None else (rank + 1) % size
    prv = dist.get_global_rank(group, (rank - 1) % size) if group is not None else (rank - 1) % size
    msg = None
    try:
        while True:
            kind, payload = gen.send(msg)
            if kind == "start":
                bufs = [torch.empty_like(t) for t in payload]
                ops = [dist.P2POp(dist.isend, t, nxt, group) for t in payload]
                ops += [dist.P2POp(dist.irecv, b, prv, group) for b in bufs]
                msg = (dist.batch_isend_irecv(ops), bufs)
            else:
                reqs, bufs = payload
                for r in reqs:
                    r.wait()
                msg = bufs
    except StopIteration as done:
        return done.value


def _run_emulated(gens):
    """Step N per-rank generators in lockstep; a shift rotates the blocks."""
    size = len(gens)
    msgs = [None] * size
    results = [None] * size
    while True:
        outgoing = [None] * size
        active = 0
        for r, g in enumerate(gens):
            if results[r] is not None:
                continue
            try:
                kind, payload = g.send(msgs[r])
            except StopIteration as done:
                results[r] = done.value
                continue
            assert kind == "start"
            outgoing[r] = payload
            active += 1
        if active == 0:
            return results
        if active != size:
            raise RuntimeError("ring ranks fell out of step")
        for r, g in enumerate(gens):
            kind, handle = g.send(r)  # the handle is just the rank index
            assert kind == "wait"
        msgs = [outgoing[(r - 1) % size] for r in range(size)]


def ring_forward(q, k, v, rope_theta=1e4, softmax_scale=0.0, group=None, ops=None):
    """This rank's block of O (dtype of q) and LSE [B, H, n] (fp32) for causal
    attention over the sequence formed by all ranks' blocks in rank order."""
    import torch.distributed as dist
    ops = ops or GpuBlockOps()
    gen = _forward_steps(dist.get_rank(group), dist.get_world_size(group), q, k, v,
                         rope_theta, softmax_scale, ops)
    return _run_distributed(gen, group)


def ring_backward(q, k, v, o, lse, d_o, rope_theta=1e4, softmax_scale=0.0, group=None, ops=None):
    """This rank's blocks of dq, dk, dv (gradients w.r.t. the un-rotated inputs)."""
    import torch.distributed as dist
    ops = ops or GpuBlockOps()
    gen = _backward_steps(dist.get_rank(group), dist.get_world_size(group), q, k, v, o, lse, d_o,
                          rope_theta, softmax_scale, ops)
    return _run_distributed(gen, group)


def emulated_ring_forward(q_blocks, k_blocks, v_blocks, rope_theta=1e4, softmax_scale=0.0,
                          ops=None):
    """The ring forward for N virtual ranks on one device (lists of blocks)."""
    ops = ops or GpuBlockOps()
    n = len(q_blocks)
    gens = [_forward_steps(r, n, q_blocks[r], k_blocks[r], v_blocks[r], rope_theta,
                           softmax_scale, ops) for r in range(n)]
    return _run_emulated(gens)


def emulated_ring_backward(q_blocks, k_blocks, v_blocks, o_blocks, lse_blocks, do_blocks,
                           rope_theta=1e4, softmax_scale=0.0, ops=None):
    ops = ops or GpuBlockOps()
    n = len(q_blocks)
    gens = [_backward_steps(r, n, q_blocks[r], k_blocks[r], v_blocks[r], o_blocks[r],
                            lse_blocks[r], do_blocks[r], rope_theta, softmax_scale, ops)
            for r in range(n)]
    return _run_emulated(gens)
