"""Host-side multi-rank logic of bench.py with 2 gloo ranks on the CPU:
max-over-ranks timing and one distinct image per rank (replicas, no
data-path collective)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    r, w, lr = bench.dist_env()
    got = bench.reduce_max(float(10 * (rank + 1)), w)
    import workloads as W
    wl = W.WORKLOADS[bench.DEFAULT_WORKLOAD]
    offs, valid = W.layout(wl, seed=777 + wl.seed_base + 1000 * rank)
    x = W.features(1, 8, 1234 + wl.seed_base + 1000 * rank)
    q.put((r, w, got, int(offs[-1]), float(x.float().sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_distinct_images():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, q), nprocs=2, join=True, start_method="spawn")
    res = sorted(q.get() for _ in range(2))
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 20.0 for r in res)          # max over ranks
    assert res[0][3] == res[1][3] == 13             # one 13-tile image per rank
    assert res[0][4] != res[1][4]                   # different data per rank


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
