"""Head-sharded SCOPE calls over the ranks of a process group.

The SCOPE abstract ("SCOPE: Subspace Clustering with Online Per-Head Top-K
Estimation for Sparse Video Attention") clusters every head on its own and
takes a head-specific Top-k: no step mixes heads.  So the heads of one call
split across GPUs with no exchange on the data path:

  * heads go round-robin: rank r of W takes heads r, r + W, r + 2W, ...;
  * every rank runs scope_plan + scope_attn on its own heads only (the
    library reads a head slice of a [B, H, N, D] tensor in place, as a
    strided view, so slicing copies nothing);
  * only a caller that needs the whole output on every rank gathers it:
    one all-gather over the head dimension (NCCL over NVLink on GPUs).

The per-rank compute is the library call by default; `run` may replace it
(the CPU tests of this module pass a host implementation, since gloo ranks
have no GPU).
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch
import torch.distributed as dist


def world_and_rank(group=None):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def heads_of(H: int, rank: int, world: int) -> List[int]:
    """Heads of rank `rank` among `world`: rank, rank + world, ..."""
    if not 0 <= rank < world:
        raise ValueError("rank outside [0, world)")
    return list(range(rank, H, world))


def local_heads(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Rank `rank`'s heads of a full [B, H, N, D] tensor, as a view."""
    return x[:, rank::world]


def run_library(q, k, v, params, grid, out=None):
    """scope_plan + scope_attn on the given heads (device tensors)."""
    import cluster_guided_sparse_b200 as scope

    pl = scope.plan(q, k, params, grid)
    return scope.attn(q, k, v, pl, out=out)


def sharded_attention(q, k, v, params, grid, H: Optional[int] = None, group=None, gather: bool = True,
                      run: Optional[Callable] = None):
    """One SCOPE call with its heads split over the ranks of `group`.

    q, k, v are either the full [B, H, N, D] tensors (every rank then takes
    its own heads as views) or this rank's heads already (pass the total head
    count as `H`).  Returns this rank's output heads, or with `gather` the
    full [B, H, N, D] output on every rank."""
    world, rank = world_and_rank(group)
    H_total = q.shape[1] if H is None else H
    mine = heads_of(H_total, rank, world)
    if q.shape[1] == H_total and world > 1:
        q, k, v = (local_heads(t, rank, world) for t in (q, k, v))
    if q.shape[1] != len(mine):
        raise ValueError(f"rank {rank} holds {q.shape[1]} heads, expected {len(mine)} of {H_total}")
    o = (run or run_library)(q, k, v, params, grid)
    if not gather or world == 1:
        return o
    return gather_heads(o, H_total, group)


def gather_heads(o_local: torch.Tensor, H: int, group=None) -> torch.Tensor:
    """Full [B, H, N, D] output from every rank's round-robin head slice:
    one all-gather of equal-sized (padded) chunks, then each rank's heads are
    put back at r, r + W, ..."""
    world, rank = world_and_rank(group)
    B, _, N, D = o_local.shape
    h_max = (H + world - 1) // world
    chunk = o_local.new_zeros((B, h_max, N, D))
    chunk[:, :o_local.shape[1]] = o_local
    parts = [torch.empty_like(chunk) for _ in range(world)]
    dist.all_gather(parts, chunk, group=group)
    out = o_local.new_empty((B, H, N, D))
    for r in range(world):
        n_r = len(heads_of(H, r, world))
        out[:, r::world] = parts[r][:, :n_r]
    return out
