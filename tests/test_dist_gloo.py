"""Host logic of the multi-rank bench path on CPU ranks (gloo, world size 2).

bench.py runs token data-parallel replicas: each rank holds the whole layer and its own
batch, the process group only carries the barrier and the max over ranks of the timing,
and rank 0 alone prints the JSON line.  These tests run that plumbing in two CPU processes.
"""

import io
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import bench
        ms = bench.reduce_max(1.0 + 2.5 * rank, world)  # the slower rank sets the job time
        rate = bench.whole_job_rate(8, world, ms)
        buf = io.StringIO()
        printed = bench.emit({"rank": rank, "ms": ms}, rank, stream=buf)
        dist.barrier()
        # the reference arm: ranks other than 0 exit without work
        class A:
            steps, warmup, gpus = 1, 0, world
        ran = False
        if rank != 0:
            bench.run_reference(A, None, rank, world)  # returns before touching the shape
            ran = True
        q.put((rank, ms, rate, printed, buf.getvalue(), ran))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_max_timing_and_rank0_output(repo_root):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, rate0, pr0, out0, _), (r1, ms1, rate1, pr1, out1, ran1) = res
    assert ms0 == ms1 == 3.5
    assert rate0 == rate1 == pytest.approx(2 * 8 / 3.5e-3)
    assert pr0 and not pr1 and '"rank": 0' in out0 and out1 == ""
    assert ran1


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max(4.25, 1) == 4.25
    assert bench.whole_job_rate(8, 1, 0.25) == pytest.approx(32000.0)
