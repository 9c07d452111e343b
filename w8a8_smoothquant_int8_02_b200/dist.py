"""Multi-process plumbing for the SmoothQuant linear layer.

The layer shards over tokens: every token row is quantized and multiplied
independently, so N GPUs run N independent problems (no collective on the
data path). Two host-side steps do exchange data:

* calibration over a corpus split across ranks: each rank reduces its shard
  with sq_calibrate_amax, then one all-reduce(MAX) of the K per-channel
  values gives every rank the amax of the whole corpus (the smoothing
  factors need max|X_j| over all calibration tokens, "Weight-Activation
  Quantization" §3 "Choosing the Smoothing Factor");
* timing: the job's time is the maximum over ranks.

torch.distributed carries both (NCCL on GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def allreduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In place: amax <- elementwise max over ranks (no-op on one process)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def shard_rows(n_rows: int, world_size: int, rank: int) -> slice:
    """Contiguous, balanced split of n_rows over ranks (sizes differ by <= 1)."""
    base, extra = divmod(n_rows, world_size)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def calibrate_activation_amax(x_cal_shard: torch.Tensor, amax_fn, group=None) -> torch.Tensor:
    """Per-channel amax of a calibration corpus spread over ranks.

    amax_fn(x) -> [K] float32 reduces one rank's [tokens, K] shard (on a GPU
    this is ops.calibrate_amax(x, "column")); an empty shard contributes
    zeros, which never change a maximum of absolute values."""
    if x_cal_shard.shape[0] == 0:
        local = torch.zeros(x_cal_shard.shape[1], dtype=torch.float32, device=x_cal_shard.device)
    else:
        local = amax_fn(x_cal_shard)
    return allreduce_amax_(local, group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest value any rank reports (job time = slowest rank)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
