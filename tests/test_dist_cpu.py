"""Multi-process (gloo, world size 2, CPU) checks of the data-parallel path:
tokens shard across ranks with no exchange, and the benchmark's per-rank
bookkeeping (seeds, max-over-ranks timing, whole-job throughput) is right."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from mixture_lookup_experts_b200 import inputs
        res = {}
        # 1. per-rank seeds differ, so ranks draw distinct batches
        seeds = bench.rank_seeds(1004, rank)
        all_seeds = [None] * world
        dist.all_gather_object(all_seeds, seeds)
        res["seeds_distinct"] = len(set(all_seeds)) == world
        # 2. the job's time is the slowest rank's; throughput counts all ranks
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank], torch.device("cpu"))
        res["max"] = mx
        res["value"] = bench.whole_job_tokens_per_s(world, 16384, 10, mx[0])
        # 3. a token batch split across ranks combines to the unsplit result
        rng = np.random.default_rng(7)
        V, D, N, T = 50, 32, 4, 40
        lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
        Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
        h = inputs.normal(rng, (T, D), 1.0, "bf16")
        ids = inputs.zipf_ids(rng, T, V)
        shard = np.array_split(np.arange(T), world)[rank]
        part, _ = oracle.combine(ids[shard], h[shard], Wr, lut, nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, part)
        full, _ = oracle.combine(ids, h, Wr, lut, nthreads=1)
        res["shards_equal"] = bool(np.array_equal(np.concatenate(parts), full))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_timing(oracle_mod):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert results[r]["seeds_distinct"]
        assert results[r]["max"] == [11.0, 5.0]
        assert results[r]["value"] == pytest.approx(2 * 16384 * 10 / 0.011)
        assert results[r]["shards_equal"]
