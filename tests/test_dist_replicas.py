"""Multi-process logic of the benchmark, on CPU with the gloo backend.

The path shards into independent (batch, KV head) units, so several GPUs run
replicas: each rank decodes its own batch of sequences and the only
collective is the max over ranks of the measured step time.  Two gloo ranks
check that every rank sees the slowest rank's time and the same whole-job
value.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_init("gloo")
    local_ms = 1.0 + 0.5 * r            # rank 1 is slower
    ms, value = bench.weak_scaling_value(local_ms, batch=8, world=w)
    bench.dist_barrier(w)
    q.put((r, ms, value))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_replicas_take_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, ms, value in res:
        assert ms == pytest.approx(1.5)
        assert value == pytest.approx(8 * world / 1.5e-3)


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.weak_scaling_value(2.0, batch=8, world=1)
    assert ms == 2.0 and value == pytest.approx(4000.0)
