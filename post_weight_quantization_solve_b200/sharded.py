"""Multi-GPU plumbing of the layer solve: one process per GPU over torch.distributed.

[GPTQ blog] "Calibration 让量化看见输入方向": H = 2 X^T X is a sum over tokens, accumulated
batch by batch, so token chunks can be summed on different GPUs and added once; and
"GPTQ 怎样把逐个补偿变成可扩展算法": every output channel is quantised independently given
the shared factor U. A layer therefore splits across N ranks as
  1. rank r accumulates its contiguous share of the token chunks into a partial H (and,
     for GPTAQ, C), with the library's Gram kernels;
  2. one all-reduce (sum) gives every rank the whole statistic (NCCL over NVLink; the
     only exchange of the solve, K^2 fp32 per statistic);
  3. every rank factors H (replicated: the factorisation is a chain of dependent panel
     steps that would need a collective per panel to split);
  4. rank r quantises its contiguous slice of output channels;
  5. where one rank needs the whole layer, an all-gather assembles codes and scales.
The helpers here are the host side of that split: which chunks and channels a rank owns
and the collectives. Every step of the solve itself runs in the library's kernels.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def chunk_range(num_chunks: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous chunk indices [c0, c1) of `rank`: sizes differ by at most one, and the
    ranks' ranges partition [0, num_chunks) in rank order (a rank may own none)."""
    if world < 1 or not 0 <= rank < world or num_chunks < 0:
        raise ValueError("need 0 <= rank < world and num_chunks >= 0")
    return num_chunks * rank // world, num_chunks * (rank + 1) // world


def channel_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous output channels [n0, n1) of `rank` (the same balanced split)."""
    return chunk_range(N, rank, world)


def channel_segments(n0: int, n1: int, N: int, groups: int = 1) -> list[tuple[int, int, int]]:
    """Split channels [n0, n1) at the output-group boundaries (group i is channels
    [i N / g, (i + 1) N / g) with its own Hessian): a list of (group, a, b) segments,
    each quantised with that group's factor."""
    if groups < 1 or N % groups:
        raise ValueError("N must be a multiple of groups")
    per = N // groups
    out = []
    a = n0
    while a < n1:
        g = a // per
        b = min(n1, (g + 1) * per)
        out.append((g, a, b))
        a = b
    return out


def allreduce_statistics(*tensors: torch.Tensor, group=None) -> None:
    """Sum each statistic (H, H_g stacks, C) over the ranks, in place."""
    for t in tensors:
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def all_gather_rows(local: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """Rows [n0, n1) of every rank (channel_range's split of N) -> the whole [N, ...].

    Slices are padded to the longest one so a single equal-size all-gather serves
    uneven splits; the padding is dropped on assembly."""
    world = dist.get_world_size(group)
    longest = max(b - a for a, b in (channel_range(N, r, world) for r in range(world)))
    pad = torch.zeros((longest,) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    rows = []
    for r in range(world):
        a, b = channel_range(N, r, world)
        rows.append(parts[r][:b - a])
    return torch.cat(rows, dim=0)


def max_over_ranks(x: torch.Tensor, group=None) -> torch.Tensor:
    """Element-wise maximum over the ranks, in place (timings: the slowest rank)."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(x, op=dist.ReduceOp.MAX, group=group)
    return x
