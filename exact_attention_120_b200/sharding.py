"""Host-side plumbing for running the forward pass on several GPUs.

Attention heads are independent problems: a forward pass has no exchange
step, so ranks never communicate on the data path.  With N ranks (one
process per GPU, launched by torchrun), rank r processes its own batch
slice of the workload's shape (its own seed, ``rank_seed``: weak scaling);
the only collectives are barriers around the timed region and a max over
ranks of the elapsed time (``timed_region``).
"""

from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world_size: int
    local_rank: int

    @property
    def is_root(self) -> bool:
        return self.rank == 0


def rank_info_from_env(env=None) -> RankInfo:
    env = os.environ if env is None else env
    return RankInfo(int(env.get("RANK", 0)), int(env.get("WORLD_SIZE", 1)),
                    int(env.get("LOCAL_RANK", env.get("RANK", 0))))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic inputs (weak scaling: each rank owns a
    different batch slice of the same shape)."""
    return int(seed) + 1000 * int(rank)


def init_process_group(info: RankInfo, backend: str, timeout_s: float = 120.0):
    import torch.distributed as dist

    if info.world_size > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, rank=info.rank, world_size=info.world_size,
                                timeout=datetime.timedelta(seconds=timeout_s))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_region(step, steps: int, timer, device=None, sync=None) -> float:
    """Time `steps` calls of `step` on every rank and return the job's time
    per step in ms: the max over ranks.

    Each rank: barrier, `sync()` (e.g. a device synchronise), `timer.start()`,
    the steps, `timer.stop()`, `sync()`, barrier; then the elapsed time
    (`timer.elapsed_ms()`) goes through one max-reduction.  Every rank takes
    the same collective steps in the same order."""
    barrier(device)
    if sync is not None:
        sync()
    timer.start()
    for _ in range(steps):
        step()
    timer.stop()
    if sync is not None:
        sync()
    barrier(device)
    return max_over_ranks(timer.elapsed_ms(), device) / steps


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def destroy():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
