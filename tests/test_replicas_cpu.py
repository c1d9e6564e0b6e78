"""The multi-process side of bench.py, on CPU with the gloo backend.

The operator needs no exchange between sequences, so N GPUs run N
independent replicas; the only collectives are the barrier around the timed
region and the max-over-ranks reduction of the measured time.  These tests run
two ranks as processes on the host (127.0.0.1) and check that the reduction
returns the slowest rank's time on every rank, that the whole-job throughput
counts every replica's tokens over that time, and that the reference arm
prints from rank 0 only.
"""
import datetime
import io
import multiprocessing as mp
import os
import socket
from contextlib import redirect_stdout

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier_sync(world, cuda=False)
        slowest = bench.max_over_ranks(1.5 + 2.0 * rank, world, device="cpu")
        bench.barrier_sync(world, cuda=False)
        out.put((rank, slowest))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(out.get(timeout=10) for _ in range(2))
    assert got == [(0, 3.5), (1, 3.5)]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.25, 1) == 2.25
    bench.barrier_sync(1, cuda=False)


def test_job_throughput_counts_every_replica_over_the_slowest_rank():
    # 4 replicas of 16,384 tokens, the slowest rank took 0.5 ms
    assert bench.job_tokens_per_s(4, 16384, 0.5) == 4 * 16384 / 0.5e-3


def test_reference_arm_prints_on_rank_zero_only():
    class Args:
        steps, warmup, gpus = 1, 1, 2
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(Args(), rank=1)
    assert buf.getvalue() == ""
