"""The multi-GPU bench path on CPU: two gloo ranks run the same barrier, max-over-ranks
timing and replica throughput that `bench.py --gpus N` uses with NCCL (replicas only: no
data-path collective)."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.0 + rank, world)          # rank r "took" 1 + r seconds
        v = bench.replica_throughput(128.0, world, t)         # 128 tokens per replica
        out.put((rank, t, v))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_replicas_slowest_rank_defines_the_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in got:
        assert t == 2.0                      # max over ranks
        assert v == pytest.approx(2 * 128.0 / 2.0)


def test_single_replica_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(128, 1, 0.5) == 256.0
