"""GPU parity of the dense comparison GEMM: the same grouped GEMM on the decoded
(dense NVFP4, pruned elements zero) weights, the pages' --no-sparse-storage form
(Usage of the MoESQ repository README), with 16-element scale blocks.

The oracle is the one of the sparse GEMM: the decoded weights and their scales are
the same numbers, so the exact grouped GEMM, the tolerance 1e-5 * sum|a w| and the
requantisation analysis carry over unchanged.
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
from oracle import formats as F
from oracle import gemm as G
from oracle import nvfp4 as N
from oracle import routing as R
from tests import parity_util as PU
from tests.parity_util import cuda
from tests.test_gpu_gemm import CASES, Layer, bf16_ulp

pytestmark = pytest.mark.gpu

TOL = 1e-5
DENSE_CASES = ["tiny", "ragged_multi_tile", "deep_k", "exact_per_half_alpha"]


def expand16(sf32):
    n = sf32.numel() // 512
    out = torch.empty(2 * n * 512, dtype=torch.uint8, device=sf32.device)
    M.moesq_sf_expand_block16(sf32, out, n)
    return out


class DenseLinear:
    """Dense codes + 16-element scale blocks of a layer's expert linear."""

    def __init__(self, storages, exp_lin):
        st = PU.storage_to_device(storages)
        E, out, K = st["E"], st["out"], st["K"]
        self.dense = torch.empty((E, out, K // 2), dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        M.moesq_decode(st["packed"], st["mask"], self.dense, E * out, K, status)
        assert int(status.item()) == 0
        self.sf16 = expand16(exp_lin.sf)
        self.alpha = exp_lin.alpha_w
        self.struct = M.Linear(self.dense.data_ptr(), 0, self.sf16.data_ptr(), self.alpha.data_ptr(), out, K, E,
                               exp_lin.kind)


@pytest.fixture(scope="module", params=DENSE_CASES)
def layer(request):
    cfg, T, *opt = CASES[request.param]
    L = Layer(cfg, T, **(opt[0] if opt else {}))
    L.dense_gu = DenseLinear(L.gu, L.dgu)
    L.dense_dn = DenseLinear(L.dn, L.ddn)
    return L


def test_sf_expand_block16_layout():
    """Expanded blocks hold, for row r and K element k, the 32-element scale of (r, k // 32),
    at the 16-element block position of (r, k // 16)."""
    rng = np.random.default_rng(5)
    rows, K = 256, 384
    sc = rng.integers(0, 256, (rows, K // 32)).astype(np.uint8)
    r = np.arange(rows)

    def blocks(s, kblk):  # per-row scales [rows, K/g] -> [rows/128][K/kblk][512]
        nb = s.shape[1] // 4
        b = np.zeros((rows // 128, nb, 512), np.uint8)
        for g in range(s.shape[1]):
            b[r // 128, g // 4, (r % 32) * 16 + ((r % 128) // 32) * 4 + g % 4] = s[:, g]
        return b.reshape(-1)

    sf32 = blocks(sc, 128)
    want = blocks(np.repeat(sc, 2, axis=1), 64)
    got = expand16(cuda(sf32)).cpu().numpy()
    assert np.array_equal(got, want)


def test_dense_gate_up_f32_within_tolerance(layer):
    L = layer
    eo, po, st, ts = L.device_routing()
    codes, sf = L.device_act(eo, po, st)
    out = torch.full((L.S, 2 * L.cfg.I), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_grouped_gemm_dense(L.dense_gu.struct, codes, expand16(sf), cuda(L.g_in_gu), eo, po, L.S, L.P, M.EPI_F32,
                               None, out, None, d_status=status)
    y = out.cpu().numpy().astype(np.float64)
    assert int(status.item()) == 0
    err = np.abs(y - L.acc_gu)
    lim = TOL * L.bound_gu + 1e-30
    assert np.isfinite(y).all()
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"


def test_dense_down_bf16_within_tolerance(layer):
    L = layer
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    rng = np.random.default_rng(3)
    h = F.bf16_round((rng.standard_normal((L.S, cfg.I)) * 2).astype(np.float32))
    g_in = L.g_in_dn
    e_of = R.slot_expert(L.perm["expert_offsets"])
    hc, hs = N.quantize_groups(h, g_in[e_of])
    yx, bound = G.grouped_gemm_exact([G.weight_int(s) for s in L.dn], [s["g"][0] for s in L.dn],
                                     G.dequant_int(hc, hs), g_in, L.perm["expert_offsets"])
    codes = torch.empty((L.P, cfg.I // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((L.P // 128) * (cfg.I // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_quant_act(cuda(h, torch.bfloat16).view(torch.uint16), cfg.I, None, eo, po, cfg.E, cuda(g_in),
                      L.S, M.SF_KERNEL, codes, sf)
    y = torch.empty((L.S, cfg.H), dtype=torch.bfloat16, device="cuda")
    M.moesq_grouped_gemm_dense(L.dense_dn.struct, codes, expand16(sf), cuda(g_in), eo, po, L.S, L.P, M.EPI_BF16,
                               None, y.view(torch.uint16), None)
    yg = y.float().cpu().numpy().astype(np.float64)
    lim = TOL * bound + bf16_ulp(yx) + 1e-30
    err = np.abs(yg - yx)
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"


def test_dense_swiglu_requant_epilogue(layer):
    L = layer
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    codes, sf = L.device_act(eo, po, st)
    h_codes = torch.empty((L.P, cfg.I // 2), dtype=torch.uint8, device="cuda")
    h_sf = torch.empty((L.P // 128) * (cfg.I // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_grouped_gemm_dense(L.dense_gu.struct, codes, expand16(sf), cuda(L.g_in_gu), eo, po, L.S, L.P,
                               M.EPI_SWIGLU_NVFP4, cuda(L.g_in_dn), h_codes, h_sf)
    got_c, got_s = PU.kernel_rows_to_slots(h_codes.cpu().numpy(), h_sf.cpu().numpy(),
                                           L.perm["expert_offsets"], L.perm["pad_offsets"], cfg.I)
    got_codes = N.unpack_codes(got_c)
    e_of = R.slot_expert(L.perm["expert_offsets"])
    an = PU.requant_analysis(G.swiglu(L.acc_gu), PU.swiglu_error_bound(L.acc_gu, L.bound_gu, TOL), L.g_in_dn[e_of])
    fixed = an["code_fixed"]
    assert np.array_equal(got_s[an["sc_fixed"]], an["sc"][an["sc_fixed"]])
    assert np.array_equal(got_codes[fixed], an["codes"][fixed])
    g = L.g_in_dn[e_of].astype(np.float64)[:, None]
    deq_gpu = F.e2m1_decode(got_codes) * np.repeat(F.e4m3_decode(got_s), 32, axis=1) * g
    deq_ref = F.e2m1_decode(an["codes"]) * np.repeat(F.e4m3_decode(an["sc"]), 32, axis=1) * g
    assert (np.abs(deq_gpu - deq_ref) <= an["max_dev"] * (1 + 1e-6) + 1e-30).all()
    assert fixed.mean() > 0.95
