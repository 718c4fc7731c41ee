"""The multi-process path on CPU: two gloo ranks exercise rank discovery, the max/sum
reductions bench.py uses for timing and throughput, and contiguous sharding."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from mask_only_logits_b200 import dist as D


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        info = D.rank_info()
        assert (info.rank, info.world, info.local_rank) == (rank, world, rank)
        dist = D.init_process_group("gloo", timeout_s=60)
        # per-rank timings: the job time is the slowest rank's
        mx = D.max_over_ranks([10.0 + rank, 5.0 - rank])
        sm = D.sum_over_ranks([1.0, float(rank)])
        # shards tile the range in rank order
        lo, hi = D.shard_range(126464, rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, mx, sm, gathered, D.replica_seed(7, rank)))
    except Exception as e:  # noqa: BLE001
        q.put((rank, repr(e)))


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        item = q.get(timeout=240)
        results[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert len(results[r]) == 5, results[r]
        _, mx, sm, gathered, seed = results[r]
        assert mx == [11.0, 5.0]
        assert sm == [2.0, 1.0]
        assert gathered == [(0, 63232), (63232, 126464)]
        assert seed == 7 + r
    assert results[0][4] != results[1][4]


def test_shard_range_properties():
    for total in (0, 1, 7, 126464, 151936):
        for world in (1, 2, 3, 8):
            shards = [D.shard_range(total, r, world) for r in range(world)]
            assert shards[0][0] == 0 and shards[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(shards, shards[1:]))
            sizes = [hi - lo for lo, hi in shards]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        D.shard_range(10, 2, 2)


def test_single_process_reductions_are_identity():
    assert D.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert D.sum_over_ranks([3.0]) == [3.0]
    assert torch.distributed.is_available()
