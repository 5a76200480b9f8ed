"""The multi-process (N > 1) host logic of bench.py on CPU: two gloo ranks
agree on the job time (the max over ranks), compute the whole-job throughput
from it, and only rank 0 runs the reference arm."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    from datetime import timedelta
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        value = bench.job_throughput(world, 16, ms)
        os.environ["RANK"] = str(rank)
        ref = bench.reference_arm(None, None) if rank != 0 else "skipped"
        q.put((rank, ms, value, ref))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value, ref in res:
        assert ms == 15.0                      # both ranks report the slower rank's time
        assert value == pytest.approx(2 * 16 / 0.015)
    assert res[1][3] is None                   # rank 1 runs no reference work


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(1, 4, 2.0) == pytest.approx(2000.0)
