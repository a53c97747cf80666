"""Multi-rank aggregation of bench.py on the CPU: two gloo ranks, no GPU.

Every (sequence, kv head) is independent, so N GPUs run N replicas and the only
cross-rank step is the timing: each rank's time goes through one all-reduce MAX and the
whole-job throughput counts every rank's bytes over the slowest rank's time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r saw step 1 + r ms, e2e 10 - r ms, attention 0.5 ms
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5], "cpu", world)
        value = bench.whole_job_gbs(world, 2e9, got[0])
        ref_args = type("A", (), {"warmup": 0, "steps": 1, "gpus": world})()
        ref = bench.run_reference(ref_args) if rank != 0 else "skipped"
        dist.barrier()
        q.put((rank, got, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_sum_bytes():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, got, value, ref = q.get(timeout=120)
        results[rank] = (got, value, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got, value, _ = results[rank]
        assert got == [2.0, 10.0, 0.5]          # max over ranks, identical on every rank
        assert value == pytest.approx(2 * 2e9 / 2e-3 / 1e9)  # 2 ranks x 2 GB in 2 ms = 2000 GB/s
    assert results[1][2] is None  # the reference arm runs on rank 0 only


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.0, 4.0], "cpu", 1) == [3.0, 4.0]
    assert bench.whole_job_gbs(1, 1e9, 1.0) == pytest.approx(1000.0)
