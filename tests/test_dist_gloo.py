"""The multi-process path on CPU: two gloo ranks exercise rank discovery, the max/sum
reductions bench.py uses for timing and throughput, contiguous sharding, and the exchange
of the vocabulary-parallel step (packed partials, one all-gather, merge in rank order)."""
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


def _shard_worker(rank: int, world: int, port: int, q):
    """One rank of a vocabulary-parallel step with the oracle standing in for the GPU
    kernels: its shard's partials, packed by PartialLayout, exchanged by exchange_partials."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import numpy as np
        import oracle.oracle as O
        import workloads as WL
        from mask_only_logits_b200.sharded import PartialLayout, exchange_partials
        D.init_process_group("gloo", timeout_s=60)
        import torch.distributed as dist
        inp = WL.make_inputs(WL.custom_config(2, 40, 32, 1001, 4, r=0.6), seed=9)
        Hb, Wb, M = WL.bf16_bits(inp["H"]), WL.bf16_bits(inp["W"]), inp["M"].numpy()
        row_idx, seq_off, count = O.mask_compact(M)
        H64 = O.bf16_bits_to_f64(Hb[row_idx])
        v0, v1 = D.shard_range(Wb.shape[0], rank, world)
        Z = O.logits_rows(H64, O.bf16_bits_to_f64(Wb[v0:v1]))
        m, s_, a = O.partial_stats(Z, 0, v1 - v0)
        lay = PartialLayout(M.size, extended=False)
        local = lay.empty(None, "cpu").fill_(float("nan"))
        f = lay.fields_of(local)
        f["m"][:count] = torch.from_numpy(m.astype(np.float32))
        f["s"][:count] = torch.from_numpy(s_.astype(np.float32))
        f["a"][:count] = torch.from_numpy((a + v0).astype(np.int32))
        gathered = lay.empty(world, "cpu")
        exchange_partials(local, gathered)
        flat = gathered.reshape(-1)
        parts = []
        for j in range(world):
            base = j * lay.split_stride
            parts.append((flat[base:base + count].double().numpy(),
                          flat[base + lay.n_pad:base + lay.n_pad + count].double().numpy(),
                          flat[base + 2 * lay.n_pad:base + 2 * lay.n_pad + count].view(torch.int32).numpy()))
        tok, _, lse, conf = O.lse_merge(parts)
        full = O.row_stats(O.logits_rows(H64, O.bf16_bits_to_f64(Wb)))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, tok.tolist() == full[0].tolist(),
               float(np.max(np.abs(lse - full[2]) / np.abs(full[2]))),
               float(np.max(np.abs(conf - full[3]) / full[3])), (v0, v1)))
    except Exception as e:  # noqa: BLE001
        q.put((rank, repr(e)))


@pytest.mark.timeout(300)
def test_vocab_sharded_exchange_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
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
        _, tok_ok, e_lse, e_conf, bounds = results[r]
        assert tok_ok
        assert e_lse < 1e-6 and e_conf < 1e-5, (e_lse, e_conf)     # fp32 packing of partials
        assert bounds == D.shard_range(1001, r, world)


def _dead_rank_worker(rank: int, world: int, port: int, q):
    """Rank 1 leaves before the step's exchange; rank 0 must get an error, not hang."""
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        from mask_only_logits_b200.sharded import PartialLayout, exchange_partials
        dist = D.init_process_group("gloo", timeout_s=5)
        dist.barrier()                                     # both ranks were up
        if rank == 1:
            q.put((rank, "left"))
            q.close()
            q.join_thread()                                # the message is out before dying
            os._exit(0)                                    # dies between steps, no goodbye
        lay = PartialLayout(64, extended=False)
        local, gathered = lay.empty(None, "cpu").zero_(), lay.empty(world, "cpu")
        t0 = time.monotonic()
        try:
            exchange_partials(local, gathered)
            q.put((rank, "no error", time.monotonic() - t0))
        except Exception as e:  # noqa: BLE001 - the collective must fail
            q.put((rank, "raised", time.monotonic() - t0, type(e).__name__))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "setup failed: " + repr(e)))


@pytest.mark.timeout(300)
def test_dead_rank_is_detected_by_the_exchange():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dead_rank_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        item = q.get(timeout=240)
        results[item[0]] = item
    for p in procs:
        p.join(timeout=60)
    assert results[1][1] == "left", results[1]
    assert results[0][1] == "raised", results[0]
    assert results[0][2] < 120.0                           # within the group's timeout budget
