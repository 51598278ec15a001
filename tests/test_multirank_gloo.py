"""Multi-rank host logic on CPU with gloo (world size 2): per-rank input
streams are disjoint, shards cover the units exactly once, and timings are
reduced with MAX over ranks."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_compression_score_b200 import dist as kd
from kv_cache_compression_score_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = kd.rank_info()
        assert (r, lr, w) == (rank, rank, world)
        # this rank's timings: rank 1 is slower on the first quantity, rank 0 on the second
        mine = [1.0 + rank, 5.0 - rank]
        mx = kd.max_over_ranks(mine)
        seed = kd.rank_seed(1002, rank)
        k, _ = synth.keys_values(seed, 0, 16, 2, 8, "f32")
        out[rank] = (mx, kd.shard_range(37, rank, world), float(k.sum()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    (mx0, sh0, s0), (mx1, sh1, s1) = out[0], out[1]
    assert mx0 == mx1 == [2.0, 5.0]
    assert sh0 == (0, 19) and sh1 == (19, 37)
    assert s0 != s1                                       # disjoint input streams
    assert kd.whole_job_rate(32768, world, 2.0) == 32768.0


def _tsp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        from oracle import kvc_oracle as O
        S, w, n_kv = 600, 32, 8
        raw = synth.random_scores(1234, (n_kv, S), 0)           # the same full [8, S] on every rank
        n_local = n_kv // world
        mine = torch.from_numpy(np.ascontiguousarray(raw[rank * n_local:(rank + 1) * n_local], dtype=np.float32))
        red = kd.tsp_exchange_raw(mine)
        idx = O.tsp_select(red.numpy().astype(np.float64), S, w, 7, 100)
        out[rank] = idx.tolist()
    finally:
        dist.destroy_process_group()


def test_tsp_head_sharded_exchange():
    """Head-sharded TSP over 2 gloo ranks: after the all-reduce of the raw rows
    every rank selects the token set the unsharded layer selects."""
    from oracle import kvc_oracle as O
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_tsp_worker, args=(world, port, out), nprocs=world, join=True)
    raw = synth.random_scores(1234, (8, 600), 0).astype(np.float32).astype(np.float64)
    ref = O.tsp_select(raw, 600, 32, 7, 100)
    assert out[0] == out[1] == ref.tolist()


def test_shard_cover_exactly_once():
    for n in (0, 1, 7, 16, 101):
        for world in (1, 2, 3, 8):
            seen = np.zeros(n, dtype=int)
            for r in range(world):
                b, e = kd.shard_range(n, r, world)
                seen[b:e] += 1
            assert np.all(seen == 1)
