"""Data-parallel plumbing for the layer: one process per GPU, tokens split across ranks.

The forward needs no exchange (each rank holds the 0.52 B/weight NF4 base and the
adapters).  The backward's one exchange is the sum of the adapter gradients over ranks:
dA = sum_ranks s (dH_r B)^T X_r and dB = sum_ranks s dH_r^T U_r, because both are sums over
tokens ("Low-Rank Adaptation (LoRA) and QLoRA: Mathematical Foundations...", section
"Gradient Dynamics and Backpropagation Mechanics": dA and dB are sums of per-token outer
products).  These helpers work with any torch.distributed backend (NCCL on GPUs, gloo on
CPU for tests).
"""
from __future__ import annotations


def token_shard(T: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of this rank's tokens when T tokens are split as evenly as possible."""
    base, extra = divmod(T, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA, dB):
    """Sum dA and dB over all ranks in place (one collective each, same order on every rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dA)
        dist.all_reduce(dB)
    return dA, dB


def backward_overlapped(grads_fn, dx_fn, grads):
    """The backward with the sum of the adapter gradients over ranks overlapping dX.

    grads_fn() enqueues dA and dB (the library's grads-only phase), which live in the one flat
    tensor `grads`; the all-reduce of `grads` is then started without waiting, dx_fn() enqueues
    dX (the library's dX-only phase) meanwhile, and the caller's stream is made to wait for the
    sum before returning.  With NCCL the reduction runs on NCCL's own stream after the gradient
    kernels and beside the dX GEMM; every rank issues the same single collective."""
    import torch.distributed as dist
    grads_fn()
    work = None
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        work = dist.all_reduce(grads, async_op=True)
    dx_fn()
    if work is not None:
        work.wait()
    return grads


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over ranks (timings are reported as the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
