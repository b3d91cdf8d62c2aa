"""The benchmark's multi-rank plumbing on CPU with world size 2 (gloo):
replicas only, so the only cross-rank steps are the barrier and the scalar
max (time) / sum (bytes) reductions that form the whole-job value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    t_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    bytes_done = 1e9 * (rank + 1)
    t_max = bench.reduce_over_ranks(t_ms, "max", w)
    b_sum = bench.reduce_over_ranks(bytes_done, "sum", w)
    value = b_sum / (t_max / 1e3) / 1e9
    q.put((rank, t_max, b_sum, value))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for rank, t_max, b_sum, value in res:
        assert t_max == 15.0 and b_sum == 3e9
        assert abs(value - 200.0) < 1e-9     # 3 GB over the slowest rank's 15 ms


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, "max", 1) == 3.5
    assert bench.reduce_over_ranks(3.5, "sum", 1) == 3.5
