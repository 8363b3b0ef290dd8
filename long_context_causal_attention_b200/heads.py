"""Head-parallel attention across GPUs: the heads of one problem split over
the ranks of a process group.

The pages' device mesh has a tensor-parallel axis (LWM research note,
"Infra": mesh dp, fsdp, tp, sp); for attention it splits the heads, and the
(batch, head) units are independent, so every rank runs the single-GPU
kernels on its own heads and the attention itself has no exchange step.  In
a model the projection before attention is column-parallel, so each rank
already holds its heads; this module gives the split and, for a harness that
starts from whole tensors, the scatter (slicing a rank's heads out) and the
gather (collecting every rank's part).  Layouts as in the C ABI: q, k, v,
dO, O and the gradients [B, S, H, D]; LSE [B, H, S].
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence, Tuple


def head_range(heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Heads [h0, h1) of `rank`: equal contiguous blocks, heads % world == 0."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if heads % world:
        raise ValueError(f"{heads} heads do not split evenly over {world} ranks")
    per = heads // world
    return rank * per, (rank + 1) * per


def scatter_heads(x, rank: int, world: int, head_dim_axis: int = 2):
    """This rank's heads of a whole tensor, contiguous (the layout the kernels
    take).  head_dim_axis: 2 for [B, S, H, D], 1 for LSE [B, H, S]."""
    h0, h1 = head_range(x.shape[head_dim_axis], rank, world)
    return x.narrow(head_dim_axis, h0, h1 - h0).contiguous()


def gather_heads(part, world: int, head_dim_axis: int = 2, group=None):
    """Every rank's part, concatenated along the head axis in rank order (an
    all-gather: each rank ends with the whole tensor)."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return part
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part.contiguous(), group=group)
    return torch.cat(parts, dim=head_dim_axis)


def run_head_parallel(step: Callable[..., Dict[str, object]], tensors: Dict[str, object],
                      rank: int, world: int, gather: bool = True, group=None,
                      names: Sequence[str] = ("q", "k", "v", "do")) -> Dict[str, object]:
    """Scatter the whole input tensors by heads, run `step` (the single-GPU
    attention of this rank's heads: keyword arguments q, k, v, do, ...) and,
    if `gather`, gather its outputs: keys "lse" along axis 1, every other
    output along axis 2."""
    local = {n: scatter_heads(tensors[n], rank, world) for n in names if tensors.get(n) is not None}
    out = step(**local)
    if not gather:
        return out
    return {key: gather_heads(val, world, 1 if key == "lse" else 2, group)
            for key, val in out.items()}
