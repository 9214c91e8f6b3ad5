"""Host logic of the multi-GPU path, on CPU with gloo (world size 2)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_120_b200 import sharding


def test_rank_info_and_seeds():
    info = sharding.rank_info_from_env({"RANK": "3", "WORLD_SIZE": "4", "LOCAL_RANK": "1"})
    assert (info.rank, info.world_size, info.local_rank, info.is_root) == (3, 4, 1, False)
    assert sharding.rank_info_from_env({}).world_size == 1
    seeds = {sharding.rank_seed(3, r) for r in range(8)}
    assert len(seeds) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _SleepTimer:
    """Wall-clock stand-in for bench.py's CUDA-event timer (same interface)."""

    def start(self):
        import time

        self.t0 = time.perf_counter()

    def stop(self):
        import time

        self.t1 = time.perf_counter()

    def elapsed_ms(self):
        return 1e3 * (self.t1 - self.t0)


def _worker(rank, world, port, out):
    """One rank of bench.py's multi-rank flow on the CPU: its own workload
    seed, the timed region through sharding.timed_region (barriers, max over
    ranks), and the JSON line printed on rank 0 only."""
    import io
    import sys
    import time

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from exact_attention_120_b200.workloads import WORKLOADS

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = sharding.RankInfo(rank, world, rank)
    sharding.init_process_group(info, "gloo", timeout_s=60)
    w = bench.rank_workload(WORKLOADS["small"], info)
    # Rank r's step takes (r + 1) x 20 ms: the job's time is rank 1's.
    ms = sharding.timed_region(lambda: time.sleep(0.02 * (rank + 1)), 3, _SleepTimer())
    seeds = [None] * world
    dist.all_gather_object(seeds, w.seed)
    buf = io.StringIO()
    printed = bench.emit(info, {"rank": rank, "ms_per_step": ms}, file=buf)
    sharding.destroy()
    out.put((rank, ms, seeds, printed, buf.getvalue()))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, seeds, printed, text in res:
        assert 40.0 <= ms < 80.0, ms  # the slower rank's 40 ms per step, on both ranks
        assert len(set(seeds)) == 2   # each rank draws its own inputs
        assert printed == (rank == 0)
        assert (text != "") == (rank == 0)
    assert res[0][1] == res[1][1]     # one max-reduced value
