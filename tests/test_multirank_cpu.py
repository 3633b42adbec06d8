"""The benchmark's multi-rank path on the CPU: two `gloo` ranks, rendezvous on 127.0.0.1.

Multi-GPU runs of the benchmark are replicas (no collective on the data path).  What
the ranks share is the timing: every rank times its own steps, the whole-job time
is the slowest rank's, and the whole-job value counts every replica's work.  The
reference arm runs on rank 0 alone; the other ranks exit without work or output.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # each rank's own total, the slowest one is the job's
        mine = 10.0 + 7.5 * rank
        res["max_ms"] = bench.max_over_ranks(mine, world, torch.device("cpu"))
        res["value"] = bench.whole_job_value(world, 4, 2e12, res["max_ms"])
        # the reference arm: ranks other than 0 do no work and print nothing
        if rank != 0:
            sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0"]
            buf = io.StringIO()
            with redirect_stdout(buf):
                res["ref_rc"] = bench.main()
            res["ref_out"] = buf.getvalue()
        dist.barrier()
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_two_rank_replica_timing_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank, args=(world, _free_port(), q), nprocs=world, join=True, start_method="spawn")
    got = dict(q.get() for _ in range(world))
    slow = 10.0 + 7.5 * (world - 1)
    for r in range(world):
        assert got[r]["max_ms"] == slow
        # 2 replicas x 4 steps x 2 TFLOP over 17.5 ms
        assert got[r]["value"] == pytest.approx(world * 4 * 2.0 / 17.5e-3)
    assert got[1]["ref_rc"] == 0 and got[1]["ref_out"] == ""


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, None) == 12.5
    assert bench.whole_job_value(1, 10, 1e12, 5.0) == pytest.approx(10 * 1.0 / 5e-3)


def test_ep_launch_count():
    """Kernels an expert-parallel step launches per rank: permute (1 kernel up to 1024
    slots, else 3), quantisation, then for received slots permute, gather, 2 GEMMs,
    gather back; and the combine."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.ep_launches(1, 8, 0) == 1 + 1 + 1
    assert bench.ep_launches(1, 8, 3) == 1 + 1 + (1 + 1 + 2 + 1) + 1
    assert bench.ep_launches(65536, 8, 524288) == 3 + 1 + (3 + 1 + 2 + 1) + 1
