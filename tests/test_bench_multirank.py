"""The multi-rank path of bench.py on CPU: two gloo ranks, max-over-ranks timing and
whole-job throughput (replicas, weak scaling: each rank runs its own layer)."""
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
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r pretends its step took (r + 1) ms and its GEMM 10 - r ms
        got = bench.max_over_ranks([1e-3 * (rank + 1), 1e-3 * (10 - rank)])
        tf = bench.whole_job_tflops(world, 2.0e9, got[0])
        q.put((rank, got, tf))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tf in res:
        assert got == pytest.approx([2e-3, 10e-3])
        # 2 ranks x 2 GFLOP in the slowest rank's 2 ms = 2 TFLOP/s for the whole job
        assert tf == pytest.approx(2.0)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_tflops(1, 1e12, 0.5) == pytest.approx(2.0)
