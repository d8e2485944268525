"""Host-side bookkeeping for running the decode on N GPUs as independent
replicas (one process per GPU; the path has no exchange step, so there is no
data-path collective).  The only collective is the timing reduction: every
rank times its own device work and the slowest rank's time is the job's.
"""
from __future__ import annotations


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of `values` (floats) over all ranks of the default
    process group; the values unchanged without one."""
    vals = [float(v) for v in values]
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return vals
    import torch

    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_rate(world: int, units_per_rank_step: float, ms_total: float, steps: int):
    """Whole-job rate (units per second) and seconds per step when each of
    `world` ranks processes `units_per_rank_step` per step and the slowest
    rank took `ms_total` milliseconds for `steps` steps."""
    if steps <= 0 or ms_total <= 0:
        raise ValueError("need a positive step count and time")
    t_step = ms_total / 1e3 / steps
    return world * units_per_rank_step / t_step, t_step
