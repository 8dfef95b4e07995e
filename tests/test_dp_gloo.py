"""Multi-rank host logic on CPU: two `gloo` ranks exercise the data-parallel
helpers that the benchmark uses after its timed region (max over ranks, status
OR) and the sequence sharding, with a per-rank oracle decode standing in for
each replica's work."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from head_latent_attention_04_b200 import dp


def test_shard_sequences_balances_and_covers():
    rng = np.random.default_rng(5)
    for world in (1, 2, 3, 8):
        for _ in range(20):
            lens = rng.integers(1, 20000, size=int(rng.integers(0, 50))).tolist()
            shards = dp.shard_sequences(lens, world)
            assert len(shards) == world
            flat = sorted(i for s in shards for i in s)
            assert flat == list(range(len(lens)))
            assert all(s == sorted(s) for s in shards)
            if lens:
                loads = [sum(lens[i] for i in s) for s in shards]
                # longest-first greedy: the gap between the heaviest and lightest
                # rank is at most the longest sequence
                assert max(loads) - min(loads) <= max(lens)


def test_shard_sequences_small_cases():
    assert dp.shard_sequences([], 2) == [[], []]
    assert dp.shard_sequences([5], 3) == [[0], [], []]
    assert dp.shard_sequences([10, 10, 10, 10], 2) == [[0, 2], [1, 3]]
    assert dp.shard_sequences([100, 1, 1, 98], 2) == [[0], [1, 2, 3]]
    with pytest.raises(ValueError):
        dp.shard_sequences([1], 0)


def test_single_process_is_identity():
    assert dp.reduce_max([1.5, 2.0]) == [1.5, 2.0]
    assert dp.reduce_status(6) == 6
    assert dp.replica_seed(1, 0) == 1 and dp.replica_seed(1, 3) == 3001


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from head_latent_attention_04_b200 import workloads as W
        from oracle import mla_oracle as O
        # each replica decodes its own batch of the same shape (weak scaling)
        w = W.preset_workload("tiny", device="cpu", seed=dp.replica_seed(0, rank))
        f64 = lambda t: t.double().numpy()
        ref = O.mla_decode(f64(w.q_nope), f64(w.q_rope), [f64(w.cache_rows(b)) for b in range(w.B)],
                           f64(w.w_uk), f64(w.w_uv), w.s_q, with_intermediates=False)
        checksum = float(np.abs(ref["out"]).sum())
        # the bookkeeping collectives, in the order the benchmark takes them
        times = dp.reduce_max([1.0 + rank, 10.0 - rank, checksum])
        status = dp.reduce_status(1 << rank)
        # strong-scaling split of one global batch: every rank computes the same shards
        shards = dp.shard_sequences([4096, 100, 7000, 64, 3000], world)
        gathered = [None] * world
        torch.distributed.all_gather_object(gathered, (shards, checksum))
        q.put((rank, times, status, gathered))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            rank, times, status, gathered = q.get(timeout=240)
            results[rank] = (times, status, gathered)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    checks = [results[0][2][r][1] for r in range(world)]
    assert checks[0] != checks[1]                     # replicas draw different batches
    for r in range(world):
        times, status, gathered = results[r]
        assert times[0] == 2.0 and times[1] == 10.0   # element-wise max over ranks
        assert times[2] == max(checks)
        assert status == 0b11                         # OR of every rank's status bits
        assert gathered[0][0] == gathered[1][0] == dp.shard_sequences([4096, 100, 7000, 64, 3000], world)
