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


def test_step_launch_count():
    """Kernels one single-GPU step launches: permute (1 kernel up to 1024 slots, else 3),
    the routed quant (plus the in-place scale rearrangement once its codes reach 64 MiB,
    when H % 1024 == 0 and k <= 32), the two GEMMs and the combine."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    C = W.CONFIGS
    assert bench.kernels_per_step(C["qwen3_235b_a22b"], 65536) == 3 + 2 + 3   # 1 GiB of codes
    assert bench.kernels_per_step(C["qwen3_30b_a3b"], 16384) == 3 + 2 + 3    # 128 MiB
    assert bench.kernels_per_step(C["qwen3_30b_a3b"], 4096) == 3 + 1 + 3     # 32 MiB
    assert bench.kernels_per_step(C["qwen3_30b_a3b"], 64) == 1 + 1 + 3      # 512 slots
    assert bench.kernels_per_step(C["kimi_k2"], 1) == 1 + 1 + 3
    assert bench.kernels_per_step(C["tiny"], 64) == 1 + 1 + 3                # H = 256


def test_fp4_peak_is_the_larger_of_microbenchmark_and_eight_bf16():
    """The GEMM roofline's sparse FP4 peak: max(measured sparse-MMA rate, 8 x bf16 burst);
    the sustained peak scales the microbenchmark by the bf16 sustained / burst ratio."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = dict(hbm_gbs=6542.4, bf16_tflops=1671.8, bf16_tflops_sustained=1410.6, source="measured")
    assert bench.fp4_peaks(peaks) == pytest.approx((8 * 1671.8, 8 * 1410.6))
    peaks["fp4sp_micro"] = 17764.0
    burst, sust = bench.fp4_peaks(peaks)
    assert burst == pytest.approx(17764.0)
    assert sust == pytest.approx(17764.0 * 1410.6 / 1671.8)
    peaks["fp4sp_micro"] = 9000.0       # a slower measurement never lowers the peak
    assert bench.fp4_peaks(peaks)[0] == pytest.approx(8 * 1671.8)
    # a row is tensor-bound when its FLOPs at the peak take longer than its bytes at HBM
    bound, t, cls, target = bench.classify(1e15, 1e9, 5e8, peaks)
    assert bound == "tensor" and cls == "prefill-sized" and target == 0.60
    bound, t, cls, target = bench.classify(1e12, 1e9, 9e8, peaks)
    assert bound == "hbm" and cls == "decode-sized" and target == 0.70
