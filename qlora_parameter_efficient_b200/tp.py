"""Row-sharded (tensor-parallel) plumbing for very large d_out: one process per GPU, rank p
holding rows [b_p, e_p) of W0 (as its own NF4 weight) and the same rows of B; X, A and U are
replicated.

"Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations...", section "Gradient
Dynamics and Backpropagation Mechanics", written per shard p of the output rows:
  H[:, b_p:e_p] = X W0_p^T + s U B_p^T                       (no exchange; gathered if needed)
  G            = sum_p dH_p B_p                              (dH_p = dH[:, b_p:e_p])
  dX           = sum_p (dH_p W0_p + s (dH_p B_p) A)          -> all-reduce of the partials
  dA           = s G^T X = sum_p s (dH_p B_p)^T X            -> all-reduce of the partials
  dB[b_p:e_p]  = s dH_p^T U                                  (local)
Each rank runs the ordinary layer calls on its shard (qlora_linear_fwd / qlora_linear_bwd with
its rows of W0 and B, its columns of dH); these helpers do the partitioning and the exchanges,
with any torch.distributed backend (NCCL on GPUs, gloo on CPU for tests).

Shard boundaries are multiples of `row_align(d_in)` rows: a multiple of 16 (so a shard's rows
stay valid for every entry point, the FP8 backward included) whose blocks fill whole 256-block
groups, so that quantizing a shard gives exactly the codes, absmax bytes and second-level
constants of those rows in the unsharded weight.
"""
from __future__ import annotations

import math

BLOCK = 64       # weights per absmax block (fixed by the stored format)
GROUP = 256      # blocks per second-level group


def row_align(d_in: int) -> int:
    """Smallest row count that is a multiple of 16 and holds a whole number of 256-block groups."""
    if d_in % BLOCK:
        raise ValueError("d_in must be a multiple of 64")
    blocks_per_row = d_in // BLOCK
    rows_per_groups = GROUP // math.gcd(GROUP, blocks_per_row)   # rows whose blocks fill groups
    return 16 * rows_per_groups // math.gcd(16, rows_per_groups)


def row_shard(d_out: int, d_in: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of this rank's output rows: aligned chunks split as evenly as possible (the
    last rank also takes the ragged remainder of d_out)."""
    a = row_align(d_in)
    chunks = -(-d_out // a)
    base, extra = divmod(chunks, world)
    c0 = rank * base + min(rank, extra)
    c1 = c0 + base + (1 if rank < extra else 0)
    return min(c0 * a, d_out), min(c1 * a, d_out)


def allgather_columns(H_shard, d_out: int, world: int):
    """H [T, d_out] from every rank's column block H[:, b_p:e_p] (same order on every rank)."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return H_shard
    T = H_shard.shape[0]
    # shard widths differ only at the ragged end: gather them, then equal-width padded blocks
    w = torch.tensor([H_shard.shape[1]], dtype=torch.int64, device=H_shard.device)
    allw = [torch.zeros_like(w) for _ in range(world)]
    dist.all_gather(allw, w)
    widths = [int(x.item()) for x in allw]
    if sum(widths) != d_out:
        raise ValueError("column shards do not add up to d_out")
    pad = torch.zeros((T, max(widths)), dtype=H_shard.dtype, device=H_shard.device)
    pad[:, :H_shard.shape[1]] = H_shard
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([p[:, :wp] for p, wp in zip(parts, widths)], dim=1)


def allreduce_partials(*tensors):
    """Sum each tensor over all ranks in place (dX and dA partials), one collective each in the
    given order on every rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        for t in tensors:
            dist.all_reduce(t)
    return tensors
