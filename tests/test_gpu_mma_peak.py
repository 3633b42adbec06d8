"""The sparse FP4 tensor-core rate measurement (moesq_measure_sparse_mma_peak), the
roofline denominator of the grouped GEMMs together with 8 x the measured bf16 GEMM
rate: it runs to completion without a timeout flag, reports a rate within the range a
B200 can reach (below 1.5 x the 18 PFLOP/s sparse FP4 figure, above a tenth of it),
a wider N is not slower per FLOP, and bad arguments are refused."""
import pytest
import torch

import sparse_nvfp4_moe_b200 as M

pytestmark = pytest.mark.gpu


def test_sparse_mma_peak_runs_and_is_plausible():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    r256 = M.moesq_measure_sparse_mma_peak(2000, 256, status)
    r128 = M.moesq_measure_sparse_mma_peak(2000, 128, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert 1800.0 < r256 < 27000.0, r256
    assert r256 >= 0.9 * r128, (r256, r128)


def test_sparse_mma_peak_arguments():
    for iters, n in ((0, 256), (10, 8), (10, 264), (10, 200)):
        with pytest.raises(M.MoesqError):
            M.moesq_measure_sparse_mma_peak(iters, n)
