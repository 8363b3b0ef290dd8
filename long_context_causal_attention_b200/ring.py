"""Sequence-parallel (ring) attention over the library's block kernels.

Blockwise RingAttention, the design the LWM pages train with (research note,
sections "模型架构" and "Infra"; paper card, Summary): the sequence of each
row is split into N equal blocks, block r held by rank r of a ring.  Every
rank keeps its query block and passes its key/value block to the next rank N
times over, so each query block meets every key/value block once; the
per-block results combine exactly by their log-sum-exp, so the result equals
attention over the whole sequence.  With a causal mask, chunk pairs whose
keys all come after the queries are skipped, the diagonal pair is causal
inside and earlier chunks are attended in full.  Token layout: "contiguous"
(rank r holds chunk r of N, so late ranks do most of the causal work) or
"zigzag" (the default: 2N chunks, rank r holds chunks r and 2N-1-r, the
same work on every rank).

Backward: every rank computes, for each visiting key/value block, the
contributions to its own dq and to the visitor's dk and dv (FlashAttention
recomputation with the GLOBAL log-sum-exp and D = dO . O, so block
contributions simply add); the visitor's dk/dv sums travel after it and are
home after N shifts.  The next key/value block is sent before the current
one is computed, so only the sums wait for the step's compute.  Block
results are fp32 where the library writes them so, so the merge and the
sums carry no per-block bf16 rounding.

Each step of the arithmetic runs in the library's CUDA kernels
(lwm_rope_apply_at, lwm_attn_fwd / lwm_attn_bwd on rotated inputs,
lwm_attn_merge, lwm_accumulate, lwm_convert_f32); this module only orders
them and moves blocks.  Two stepping loops run the same per-rank algorithm:
``ring_forward`` / ``ring_backward`` for one rank of a torch.distributed
process group (NCCL point-to-point over NVLink; block i+1 is in flight while
block i is computed), and ``emulated_ring_forward`` / ``..._backward`` for
N virtual ranks stepped in lockstep on one device (same kernels, the shift
is a rotation of a list).  Packed rows: the segment ids of each rank's
chunks (cut like q) travel with the key blocks, and every block pair is
masked by query ids against key ids (lwm_attn_fwd_pair / lwm_attn_bwd_pair).
"""
from __future__ import annotations

import torch

from . import _lib as L


class GpuBlockOps:
    """Per-block operations of the ring, on the library's kernels.  Block
    results come back in fp32 where the library can write them so (fp32
    inputs; bf16 at head_dim 128 on the tensor cores), so the merge and the
    gradient sums see no per-block bf16 rounding; other shapes fall back to
    results in the input dtype."""

    def __init__(self):
        self.f32 = True

    def rotate(self, x, theta, pos0, inverse=False):
        return L.lwm_rope_apply_at(x, theta, pos0, inverse)

    def _try_f32(self, f32_call, call):
        if self.f32:
            try:
                return f32_call()
            except L.LwmError as e:
                if e.status != -2:  # anything but LWM_ERR_UNSUPPORTED is an error
                    raise
                self.f32 = False
        return call()

    def block_fwd(self, q, k, v, causal, scale, q_seg=None, k_seg=None):
        # inputs are rotated already: rope_theta = 0
        return self._try_f32(
            lambda: L.lwm_attn_fwd_pair_f32(q, k, v, q_seg, k_seg, causal, 0.0, scale),
            lambda: L.lwm_attn_fwd_pair(q, k, v, q_seg, k_seg, causal, 0.0, scale))

    def block_bwd(self, q, k, v, o, lse, d_o, causal, scale, q_seg=None, k_seg=None):
        return self._try_f32(
            lambda: L.lwm_attn_bwd_pair_f32(q, k, v, o, lse, d_o, q_seg, k_seg, causal, 0.0, scale),
            lambda: L.lwm_attn_bwd_pair(q, k, v, o, lse, d_o, q_seg, k_seg, causal, 0.0, scale))

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
# token layout: which global chunks of the sequence each rank holds
# ----------------------------------------------------------------------------
def chunk_ids(rank: int, size: int, layout: str):
    """Global chunk indices held by ``rank``, in the order they sit in its
    local tensors.  "contiguous": N chunks, rank r holds chunk r.  "zigzag":
    2N chunks, rank r holds chunks r and 2N-1-r, so every rank has the same
    causal work (an early chunk with few keys and a late one with many)."""
    if layout == "contiguous":
        return [rank]
    if layout == "zigzag":
        return [rank, 2 * size - 1 - rank]
    raise ValueError(f"unknown layout {layout!r}")


def split_for_ranks(x, size: int, layout: str = "zigzag", dim: int = 1):
    """The local tensor of every rank, cut from a whole-sequence tensor."""
    n_chunks = size * len(chunk_ids(0, size, layout))
    chunks = torch.chunk(x, n_chunks, dim=dim)
    if len({c.shape[dim] for c in chunks}) != 1 or len(chunks) != n_chunks:
        raise ValueError("sequence length must split into equal chunks")
    return [torch.cat([chunks[g] for g in chunk_ids(r, size, layout)], dim=dim).contiguous()
            for r in range(size)]


def merge_from_ranks(parts, layout: str = "zigzag", dim: int = 1):
    """Inverse of split_for_ranks: the whole-sequence tensor."""
    size = len(parts)
    per = len(chunk_ids(0, size, layout))
    chunks = [None] * (size * per)
    for r, t in enumerate(parts):
        for c, piece in zip(chunk_ids(r, size, layout), torch.chunk(t, per, dim=dim)):
            chunks[c] = piece
    return torch.cat(chunks, dim=dim)


def _pairs(q_ids, k_ids):
    """(local query chunk, visiting key chunk, causal) for every pair with
    allowed keys: earlier key chunks in full, the same chunk causally."""
    out = []
    for a, qa in enumerate(q_ids):
        for b, kb in enumerate(k_ids):
            if kb <= qa:
                out.append((a, b, kb == qa))
    return out


# ----------------------------------------------------------------------------
# the per-rank algorithm, as generators: ("start", tensors) hands the
# stepping loop the tensors to pass on to the next rank and gets back a
# handle; ("wait", handle) returns the tensors received from the previous rank.
# ----------------------------------------------------------------------------
def _forward_steps(rank, size, q, k, v, theta, scale, ops, layout, seg=None):
    ids = chunk_ids(rank, size, layout)
    c = len(ids)
    qs = torch.chunk(q, c, dim=1)
    n = qs[0].shape[1]
    B, _, H, D = q.shape
    qr = [ops.rotate(x.contiguous(), theta, g * n) for x, g in zip(qs, ids)]
    qseg = [x.contiguous() for x in torch.chunk(seg, c, dim=1)] if seg is not None else [None] * c
    # the travelling block: rotated keys, values (and the keys' segment ids)
    blk = [ops.rotate(x.contiguous(), theta, g * n) for x, g in zip(torch.chunk(k, c, 1), ids)]
    blk += [x.contiguous() for x in torch.chunk(v, c, dim=1)]
    if seg is not None:
        blk += qseg
    o_acc = [ops.zeros_f32((B, n, H, D), q.device) for _ in ids]
    lse_acc = [ops.full_f32((B, H, n), float("-inf"), q.device) for _ in ids]
    for s in range(size):
        src = (rank - s) % size
        h = (yield ("start", blk)) if s < size - 1 else None
        for a, b, causal in _pairs(ids, chunk_ids(src, size, layout)):
            kseg = blk[2 * c + b] if seg is not None else None
            o_p, lse_p = ops.block_fwd(qr[a], blk[b], blk[c + b], causal, scale, qseg[a], kseg)
            ops.merge(o_acc[a], lse_acc[a], o_p, lse_p)
        if s < size - 1:
            blk = yield ("wait", h)
    o = torch.cat([ops.convert(x, q.dtype) for x in o_acc], dim=1)
    return o, torch.cat(lse_acc, dim=2)


def _backward_steps(rank, size, q, k, v, o, lse, d_o, theta, scale, ops, layout, seg=None):
    ids = chunk_ids(rank, size, layout)
    c = len(ids)
    n = q.shape[1] // c
    B, _, H, D = q.shape
    cut = lambda t, dim=1: [x.contiguous() for x in torch.chunk(t, c, dim=dim)]
    qr = [ops.rotate(x, theta, g * n) for x, g in zip(cut(q), ids)]
    os_, dos, lses = cut(o), cut(d_o), cut(lse, 2)
    qseg = cut(seg) if seg is not None else [None] * c
    dq_acc = [ops.zeros_f32((B, n, H, D), q.device) for _ in ids]
    # the travelling block: rotated keys, values (and the keys' segment ids);
    # its gradient sums travel as a second message, sent once this rank has
    # added its contributions
    blk = [ops.rotate(x, theta, g * n) for x, g in zip(cut(k), ids)] + cut(v)
    if seg is not None:
        blk += qseg
    sums = [ops.zeros_f32((B, n, H, D), q.device) for _ in range(2 * c)]
    sums_h = None
    for s in range(size):
        src = (rank - s) % size
        # the next block is in flight while this one is computed
        kv_h = (yield ("start", blk)) if s < size - 1 else None
        parts = []
        for a, b, causal in _pairs(ids, chunk_ids(src, size, layout)):
            kseg = blk[2 * c + b] if seg is not None else None
            dq_p, dk_p, dv_p = ops.block_bwd(qr[a], blk[b], blk[c + b], os_[a], lses[a], dos[a],
                                             causal, scale, qseg[a], kseg)
            ops.accumulate(dq_acc[a], dq_p)
            parts.append((b, dk_p, dv_p))
        # the visiting block's sums, from the previous rank after its own step
        if s > 0:
            sums = yield ("wait", sums_h)
        for b, dk_p, dv_p in parts:
            ops.accumulate(sums[b], dk_p)
            ops.accumulate(sums[c + b], dv_p)
        # N shifts of the sums in all: after the last one every block's sums
        # are home
        sums_h = yield ("start", sums)
        if s < size - 1:
            blk = yield ("wait", kv_h)
    sums = yield ("wait", sums_h)
    dq = torch.cat([ops.convert(ops.rotate(x, theta, g * n, inverse=True), q.dtype)
                    for x, g in zip(dq_acc, ids)], dim=1)
    dk = torch.cat([ops.convert(ops.rotate(sums[b], theta, g * n, inverse=True), k.dtype)
                    for b, g in enumerate(ids)], dim=1)
    dv = torch.cat([ops.convert(sums[c + b], v.dtype) for b in range(c)], dim=1)
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
    """Step N per-rank generators in lockstep, one operation at a time (every
    rank runs the same sequence of starts and waits); a start records each
    rank's payload under a new handle, a wait hands every rank the payload
    its previous rank started under that handle (a shift of the ring)."""
    size = len(gens)
    msgs = [None] * size
    results = [None] * size
    in_flight, next_handle = {}, 0
    while True:
        ops_ = []
        for r, g in enumerate(gens):
            try:
                ops_.append(g.send(msgs[r]))
            except StopIteration as done:
                results[r] = done.value
                ops_.append(None)
        if all(o is None for o in ops_):
            return results
        if any(o is None for o in ops_) or len({o[0] for o in ops_}) != 1:
            raise RuntimeError("ring ranks fell out of step")
        if ops_[0][0] == "start":
            in_flight[next_handle] = [o[1] for o in ops_]
            msgs = [next_handle] * size
            next_handle += 1
        else:
            sent = in_flight.pop(ops_[0][1])
            msgs = [sent[(r - 1) % size] for r in range(size)]


def ring_forward(q, k, v, rope_theta=1e4, softmax_scale=0.0, group=None, ops=None,
                 layout="zigzag", segment_ids=None):
    """This rank's part of O (dtype of q) and LSE [B, H, n] (fp32) for causal
    attention over the whole sequence; the rank holds the chunks
    ``chunk_ids(rank, size, layout)`` (see split_for_ranks)."""
    import torch.distributed as dist
    ops = ops or GpuBlockOps()
    gen = _forward_steps(dist.get_rank(group), dist.get_world_size(group), q, k, v,
                         rope_theta, softmax_scale, ops, layout, segment_ids)
    return _run_distributed(gen, group)


def ring_backward(q, k, v, o, lse, d_o, rope_theta=1e4, softmax_scale=0.0, group=None,
                  ops=None, layout="zigzag", segment_ids=None):
    """This rank's parts of dq, dk, dv (gradients w.r.t. the un-rotated inputs)."""
    import torch.distributed as dist
    ops = ops or GpuBlockOps()
    gen = _backward_steps(dist.get_rank(group), dist.get_world_size(group), q, k, v, o, lse, d_o,
                          rope_theta, softmax_scale, ops, layout, segment_ids)
    return _run_distributed(gen, group)


def emulated_ring_forward(q_blocks, k_blocks, v_blocks, rope_theta=1e4, softmax_scale=0.0,
                          ops=None, layout="zigzag", seg_blocks=None):
    """The ring forward for N virtual ranks on one device (lists of the ranks'
    local tensors, as split_for_ranks cuts them)."""
    ops = ops or GpuBlockOps()
    n = len(q_blocks)
    gens = [_forward_steps(r, n, q_blocks[r], k_blocks[r], v_blocks[r], rope_theta,
                           softmax_scale, ops, layout,
                           seg_blocks[r] if seg_blocks is not None else None) for r in range(n)]
    return _run_emulated(gens)


def emulated_ring_backward(q_blocks, k_blocks, v_blocks, o_blocks, lse_blocks, do_blocks,
                           rope_theta=1e4, softmax_scale=0.0, ops=None, layout="zigzag",
                           seg_blocks=None):
    ops = ops or GpuBlockOps()
    n = len(q_blocks)
    gens = [_backward_steps(r, n, q_blocks[r], k_blocks[r], v_blocks[r], o_blocks[r],
                            lse_blocks[r], do_blocks[r], rope_theta, softmax_scale, ops, layout,
                            seg_blocks[r] if seg_blocks is not None else None)
            for r in range(n)]
    return _run_emulated(gens)
