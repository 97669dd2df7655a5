"""Host side of running the path as one independent replica per GPU.

The method has no exchange step between GPUs: every rank runs the whole
attention call on its own inputs (weak scaling), so the only cross-rank
traffic is timing -- a barrier around the timed region and the maximum of
the per-rank device times, which is the job's time.  These helpers hold that
logic so it can be exercised with the gloo backend on CPU as well as with
NCCL on GPUs; no attention arithmetic lives here.
"""
from __future__ import annotations

import os


def rank_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    def _i(name: str, default: int) -> int:
        try:
            return int(os.environ.get(name, default))
        except ValueError:
            return default
    return _i("RANK", 0), _i("WORLD_SIZE", 1), _i("LOCAL_RANK", 0)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity when
    torch.distributed is not initialised).  Every rank must call it with the
    same number of values, in the same order."""
    import torch
    import torch.distributed as dist
    vals = [float(x) for x in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu().tolist()]


def job_throughput(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job rate: the units every rank processed, over the slowest rank's
    time (ms), per second."""
    if ms <= 0:
        raise ValueError("time must be positive")
    return world * units_per_rank / (ms * 1e-3)
