"""Multi-process plumbing of the benchmark's replica mode, on CPU with gloo.

The hot path does not shard: N GPUs run N independent replicas (one batch
each, no data-path collective).  What crosses ranks is only the timing --
a barrier around the timed region and the maximum of the per-rank times --
and the whole-job throughput computed from it.  These tests run that
plumbing as two gloo ranks on the host.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        sys.path.insert(0, ROOT)
        import datetime
        import torch.distributed as dist
        import bench
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        assert bench.dist_env() == (rank, world, rank)
        bench.barrier(world)
        # rank r "took" 10 + r ms: every rank must see the slowest, 10 + world - 1
        slowest = bench.max_over_ranks(10.0 + rank, world)
        value = bench.replica_value(16, world, slowest)
        bench.barrier(world)
        dist.destroy_process_group()
        q.put((rank, slowest, value))
    except Exception as exc:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(exc)))


@pytest.mark.parametrize("world", [2])
def test_replica_timing_is_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in out:
        assert slowest != "error", value
        assert slowest == 10.0 + world - 1
        # 16 tokens per replica per step, `world` replicas, 11 ms per step
        assert value == pytest.approx(16 * world / (slowest / 1e3))


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_value(16, 1, 2.0) == pytest.approx(8000.0)
