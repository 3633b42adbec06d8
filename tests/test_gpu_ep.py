"""Expert parallelism with the library's kernels on one GPU (a one-rank NCCL group):
the dispatch (slot-major NVFP4 quantisation, a second permutation, the gather into the
padded operand layout) and the combine (row gather back, weighted sum) must give the
single-GPU forward's output bit for bit."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import sparse_nvfp4_moe_b200 as M
from sparse_nvfp4_moe_b200.ep import DeviceCompute, ExpertParallelMoE
from tests.parity_util import cuda
from tests.test_gpu_gemm import CASES, Layer

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("case", ["tiny", "ragged_multi_tile", "sparse_routing"])
def test_one_rank_expert_parallel_equals_forward(case):
    cfg, T, *opt = CASES[case]
    L = Layer(cfg, T, **(opt[0] if opt else {}))
    moe = M.MoELayer(cfg.k, L.dgu, L.ddn, cuda(L.g_in_gu), cuda(L.g_in_dn))
    x, ids, w = L.x.cuda(), cuda(L.ids.astype(np.int32)), cuda(L.w)
    want = moe.forward(x, ids, w)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ep = ExpertParallelMoE(cfg.E, cfg.k, cfg.H, DeviceCompute(moe, cuda(L.g_in_gu)))
        got = ep.forward(x, ids, w)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(got, want)
