"""Data-parallel plumbing for the scan: batch rows are independent problems, so ranks split the
batch with no exchange on the data path; the only cross-rank step is the sum of the parameter
gradients over (batch, time) -- dA_log [D, N] and dD [D], plus dw [D, R] and dbias [D] when the
step-size projection runs, or dlambda, domega [K] in the complex mode -- done with one all-reduce
of a packed buffer.  Works with any torch.distributed backend (NCCL on GPUs, gloo on CPU)."""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [lo, hi) range of batch rows owned by `rank` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    base, extra = divmod(int(batch), int(world))
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def allreduce_grads(grads, group=None, buf: torch.Tensor | None = None):
    """Sum every tensor of `grads` (same dtype and device) over the ranks of `group` in place,
    with one collective on a packed buffer (`buf`, reused when given, at least the total size)."""
    grads = list(grads)
    total = sum(g.numel() for g in grads)
    if buf is None:
        buf = torch.empty(total, dtype=grads[0].dtype, device=grads[0].device)
    flat = buf[:total]
    o = 0
    for g in grads:
        flat[o:o + g.numel()].copy_(g.reshape(-1))
        o += g.numel()
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    o = 0
    for g in grads:
        g.copy_(flat[o:o + g.numel()].view_as(g))
        o += g.numel()
    return grads


def allreduce_param_grads(dA_log: torch.Tensor, dD: torch.Tensor, group=None,
                          buf: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Sum dA_log and dD over the ranks of `group` in place, with one collective."""
    allreduce_grads((dA_log, dD), group=group, buf=buf)
    return dA_log, dD
