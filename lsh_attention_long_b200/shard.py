"""One problem's (batch, head) pairs split over the ranks of a process group.

Every step of LSH attention stays inside one (b, h) head: the hash, the sort
of each (round, batch, head) row, the chunked attention and the round combine
never mix heads ("Reformer explainer", akshathtiwari.co.in/blog/reformer:
attention within sorted buckets of one sequence; the definition's step 2
sorts each (batch, head, round) row on its own).  So the B*H heads of a
problem split into contiguous slices, one per rank, and each rank runs the
whole forward on its slice with no exchange on the data path.  An optional
all-gather (NCCL over NVLink on GPUs, gloo on CPUs) then puts the full O and
lse on every rank for a caller that wants them in one place.

Heads are contiguous in the [B, H, L, d] layout, so a rank's slice of the
flattened B*H heads is a plain view: no copy on the way in.
"""

from __future__ import annotations

from typing import Callable, Dict, Tuple

import torch


def head_range(n_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """[h0, h1) of the flattened B*H heads that `rank` takes: contiguous
    slices whose sizes differ by at most one, earlier ranks taking the larger."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(n_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_slice(t: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's heads of a [B, H, ...] tensor as a [1, h1 - h0, ...] view."""
    B, H = t.shape[:2]
    h0, h1 = head_range(B * H, world, rank)
    return t.reshape(1, B * H, *t.shape[2:])[:, h0:h1]


def all_gather_heads(local: torch.Tensor, B: int, H: int, world: int, rank: int,
                     group=None) -> torch.Tensor:
    """Reassembles [B, H, ...] from every rank's [1, h1 - h0, ...] slice.
    Slices are padded to the largest one so that one all_gather of equal
    sizes serves (NCCL and gloo both take it).  A world of one rank holds
    every head already and needs no process group."""
    tail = tuple(local.shape[2:])
    if world == 1:
        return local.reshape((B, H) + tail)
    import torch.distributed as dist
    per = -(-(B * H) // world)
    pad = torch.zeros((per,) + tail, dtype=local.dtype, device=local.device)
    pad[:local.shape[1]] = local[0]
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    parts = []
    for r in range(world):
        h0, h1 = head_range(B * H, world, r)
        parts.append(bufs[r][:h1 - h0])
    return torch.cat(parts, 0).reshape((B, H) + tail)


def forward_sharded(Q: torch.Tensor, V: torch.Tensor, rot: torch.Tensor, n_buckets: int,
                    chunk: int, causal: bool, world: int, rank: int,
                    forward: Callable[..., Dict[str, torch.Tensor]] = None,
                    gather: bool = False, group=None) -> Dict[str, torch.Tensor]:
    """The forward of this rank's heads of one problem.

    Returns O [1, nh, L, d] and lse [1, nh, L] of the slice (plus keys and
    perm [R, 1, nh, L]); with gather=True, also O_full [B, H, L, d] and
    lse_full [B, H, L] assembled over the group.  `forward` is the
    single-device forward to run on the slice (default: the CUDA library's
    lsh_forward); rotations are per round and shared by every head, so each
    rank uses them whole."""
    if forward is None:
        from .lsh import lsh_forward as forward
    B, H = Q.shape[:2]
    q = head_slice(Q, world, rank).contiguous()
    v = head_slice(V, world, rank).contiguous()
    out = dict(forward(q, v, rot, n_buckets, chunk, causal))
    if gather:
        out["O_full"] = all_gather_heads(out["O"], B, H, world, rank, group)
        out["lse_full"] = all_gather_heads(out["lse"], B, H, world, rank, group)
    return out
