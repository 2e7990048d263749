"""The multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing aggregation, and the
head split of one layer (each rank runs the path on its share of the heads; the shares put
back together equal the whole layer, with no collective on the data path)."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], dist, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, vals))


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 3.0]


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1, 2.5]) == [1.0, 2.5]


def _head_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np

    from free_sparse_attention_reuse_b200 import api, workload
    from helpers import oracle_anchor
    wl = workload.custom("split", 1, 5, 64, (2, 8, 16), 64, index=71)  # 5 heads over 2 ranks
    Q, K, V = workload.make_qkv(wl)
    lo, hi = api.head_shard(wl.B * wl.H, rank, world)
    # this rank's heads only (the fp64 oracle stands in for the GPU kernels here)
    mine = oracle_anchor(Q[:, lo:hi], K[:, lo:hi], V[:, lo:hi], wl.C, 100)
    parts = [None] * world
    dist.all_gather_object(parts, (lo, hi, {k: v for k, v in mine.items() if k in ("perm", "idx", "R")}))
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        whole = oracle_anchor(Q, K, V, wl.C, 100)
        ok = sorted((a, b) for a, b, _ in parts) == [(0, 3), (3, 5)]
        for a, b, m in parts:
            for key in ("perm", "idx", "R"):
                ok = ok and np.array_equal(m[key], whole[key][:, a:b])
        q.put(ok)


def test_head_split_two_gloo_ranks_reassembles_the_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok


def test_head_shard_covers_every_head_once():
    sys.path.insert(0, ROOT)
    from free_sparse_attention_reuse_b200 import api
    for n in (1, 5, 24, 40):
        for world in (1, 2, 3, 8):
            shards = [api.head_shard(n, r, world) for r in range(world)]
            assert shards[0][0] == 0 and shards[-1][1] == n
            assert all(shards[i][1] == shards[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in shards) - min(b - a for a, b in shards) <= 1
