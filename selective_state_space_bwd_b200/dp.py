"""Data-parallel plumbing for the scan: batch rows are independent problems, so ranks split the
batch with no exchange on the data path; the only cross-rank step is the sum of the parameter
gradients dA_log [D, N] and dD [D] over (batch, time), done with one all-reduce of a packed
buffer.  Works with any torch.distributed backend (NCCL on GPUs, gloo on CPU)."""

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


def allreduce_param_grads(dA_log: torch.Tensor, dD: torch.Tensor, group=None,
                          buf: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Sum dA_log and dD over the ranks of `group` in place, with one collective."""
    n = dA_log.numel()
    if buf is None:
        buf = torch.empty(n + dD.numel(), dtype=dA_log.dtype, device=dA_log.device)
    buf[:n].copy_(dA_log.reshape(-1))
    buf[n:].copy_(dD.reshape(-1))
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    dA_log.copy_(buf[:n].view_as(dA_log))
    dD.copy_(buf[n:].view_as(dD))
    return dA_log, dD
