"""Global expert load for data-parallel replicas.

The bias rule of "DeepSeek-V3 技術報告" (section 方法 / 2) reads each
expert's load over the whole step.  With one replica per GPU, every rank
routes its own tokens; the load of the step is the sum of the ranks' per-expert
counts, and the mean load uses the ranks' total token count.  This is the one
exchange the data-parallel layer needs: an all-reduce of N_r int32 counts
(NCCL on GPUs), after which every rank applies the same bias update and the
bias vectors stay identical across ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_load(counts: torch.Tensor, T_local: int, group=None, T_total: int | None = None):
    """Returns (global counts, global token count); `counts` is not modified.
    Pass T_total when every rank already knows it (equal batches): the
    counts all-reduce then stays asynchronous on the device."""
    g = counts.clone()
    dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    if T_total is not None:
        return g, T_total
    t = torch.tensor([T_local], dtype=torch.int64, device=counts.device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return g, int(t.item())
