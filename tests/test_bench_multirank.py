"""The benchmark's multi-rank bookkeeping on CPU: two `gloo` ranks.

With N GPUs the benchmark runs one independent replica per rank (the decode
path has no exchange step).  What has to be right is the bookkeeping around
the replicas: the whole-job throughput is the bytes of all ranks over the
slowest rank's time, every rank takes the same collective steps, and the
reference arm prints from rank 0 only.  These run as two spawned processes on
the host (no GPU), rendezvous on 127.0.0.1.
"""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r moved (r + 1) * 1e9 bytes in (2 + r) ms
        total, span_ms, gbs = bench.aggregate((rank + 1) * 1e9, 2.0 + rank, 2)
        bench.barrier(2)
        mx = bench.max_over_ranks(float(rank), 2)
        sm = bench.sum_over_ranks(1.0, 2)
        q.put((rank, total, span_ms, gbs, mx, sm))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregate_and_collectives():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, total, span_ms, gbs, mx, sm in res:
        assert total == pytest.approx(3e9)           # bytes of both ranks
        assert span_ms == pytest.approx(3.0)         # the slower rank's time
        assert gbs == pytest.approx(3e9 / 3e-3 / 1e9)
        assert mx == 1.0 and sm == 2.0


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(5e8, 4.0, 1) == (5e8, 4.0, pytest.approx(5e8 / 4e-3 / 1e9))
    assert bench.max_over_ranks(7.0, 1) == 7.0


def test_reference_arm_prints_from_rank0_only():
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    args = argparse.Namespace(workload="tiny_f32", steps=1, warmup=0, cpu_seconds=0.1)
    assert bench.run_reference(args, rank=1, world=2) is None
