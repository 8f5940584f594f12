"""Multi-process path of bench.py on CPU (gloo, world size 2).

The decode path needs no exchange between GPUs, so N GPUs run N independent
replicas; the only cross-rank step is taking the slowest rank's step time and
reporting N replicas' work over it.  This runs that code with two gloo ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        local_ms = 0.10 + 0.05 * rank  # rank 1 is slower
        step = bench.max_over_ranks(local_ms)
        out.put((rank, step, bench.whole_job_tflops(1e12, world, step)))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_sets_the_step_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, step, value in res:
        assert step == pytest.approx(0.15)
        assert value == pytest.approx(2 * 1e12 / 0.15e-3 / 1e12)


def test_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(0.42) == 0.42
    assert bench.whole_job_tflops(2e12, 1, 1.0) == pytest.approx(2000.0)  # 2e12 flop in 1 ms
