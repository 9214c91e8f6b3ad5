"""Host logic of the multi-GPU path, on CPU with gloo (world size 2)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_120_b200 import sharding


def test_shard_units_partition():
    for total in (0, 1, 7, 16, 33):
        for world in (1, 2, 3, 8):
            parts = [sharding.shard_units(total, world, r) for r in range(world)]
            flat = [u for p in parts for u in p]
            assert flat == list(range(total))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharding.shard_units(4, 2, 2)


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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = sharding.RankInfo(rank, world, rank)
    sharding.init_process_group(info, "gloo", timeout_s=60)
    sharding.barrier()
    # Each rank times its own shard; the job time is the max over ranks.
    t = sharding.max_over_ranks(10.0 + rank)
    units = list(sharding.shard_units(32, world, rank))
    gathered = [None] * world
    dist.all_gather_object(gathered, units)
    sharding.destroy()
    out.put((rank, t, gathered))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, gathered in res:
        assert t == 11.0  # max over ranks
        assert sorted(u for part in gathered for u in part) == list(range(32))
