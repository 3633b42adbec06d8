"""GPU parity of the grouped sparse NVFP4 GEMM, its fused SwiGLU+requant
epilogue and the whole expert MLP against the oracle.

Tolerance (per output element, float32 before output rounding):
    |y_gpu - y_exact| <= 1e-5 * sum_k |a_k w_k|        (globals applied)
and bf16 outputs within one bf16 ulp of the exact value beyond that.  The
exact value is the oracle's int64 sum (paired-4:8 NVFP4 weights, E4M3 per-32
scales, FP32 globals: "Compression details" table of the Qwen3.5-397B-A17B-
P48NVFP4-MoESQ model card).
"""
import numpy as np
import pytest
import torch

import sparse_nvfp4_moe_b200 as M
import workloads as W
from oracle import formats as F
from oracle import gemm as G
from oracle import nvfp4 as N
from oracle import routing as R
from oracle import storage as S
from tests import parity_util as PU
from tests.parity_util import cuda

pytestmark = pytest.mark.gpu

TOL = 1e-5


def bf16_ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


class Layer:
    """A small synthetic layer: oracle storage on the host, device copies repacked by the GPU."""

    def __init__(self, cfg, T, g_down_scale=1.0, routing=None, exact=False):
        """exact: gate_up with its own up global (kind GATE_UP_EXACT) instead of the fold."""
        self.cfg, self.T, self.exact = cfg, T, exact
        n_seg = 2 if cfg.split_gate_up_global else 1
        wgu = W.all_expert_weights_bf16(cfg, "gate_up")
        wdn = W.all_expert_weights_bf16(cfg, "down")
        self.gu = [S.quantize_weight(wgu[e].float().numpy(), n_seg) for e in range(cfg.E)]
        self.dn = [S.quantize_weight(wdn[e].float().numpy(), 1) for e in range(cfg.E)]
        kind_gu = (M.KIND_GATE_UP_EXACT if exact else M.KIND_GATE_UP_SPLIT) if n_seg == 2 else M.KIND_GATE_UP
        self.dgu = M.ExpertLinear.from_storage(PU.storage_to_device(self.gu), kind_gu)
        self.ddn = M.ExpertLinear.from_storage(PU.storage_to_device(self.dn), M.KIND_DOWN)
        self.x = W.layer_input_bf16(cfg, T)
        if routing is None:
            ids, w = W.routing(cfg, T)
            self.ids, self.w = ids.numpy(), w.numpy()
        else:                                   # a given [T, k] routing (ids int, weights f32)
            self.ids = np.asarray(routing[0], np.int64).reshape(T, cfg.k)
            self.w = np.asarray(routing[1], np.float32).reshape(T, cfg.k)
        self.perm = R.permute(self.ids, cfg.E)
        self.S = T * cfg.k
        self.P = M.padded_rows(self.S, cfg.E)
        self.g_in_gu = np.full(cfg.E, W.activation_global_scale_input(self.x), np.float32)
        # exact gate_up for the down-input calibration (oracle only)
        a_c, a_s = G.quant_act(self.x.float().numpy(), self.perm["slot_token"], self.perm["expert_offsets"],
                               self.g_in_gu)
        self.A = G.dequant_int(a_c, a_s)
        self.acc_gu, self.bound_gu = G.gate_up_exact(self.gu, self.A, self.g_in_gu, self.perm["expert_offsets"],
                                                     fold=not exact)
        self.g_in_dn = (PU.calibrate_g_in_down(self.acc_gu, self.perm["expert_offsets"], cfg.E) *
                        np.float32(g_down_scale)).astype(np.float32)

    def device_routing(self):
        cfg = self.cfg
        eo = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
        po = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
        st = torch.empty(self.S, dtype=torch.int32, device="cuda")
        ts = torch.empty(self.S, dtype=torch.int32, device="cuda")
        n = M.permute_workspace_size(self.T, cfg.k, cfg.E)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
        M.moesq_permute(cuda(self.ids.astype(np.int32)), self.T, cfg.k, cfg.E, eo, po, st, ts, ws, n)
        return eo, po, st, ts

    def device_act(self, eo, po, st):
        cfg = self.cfg
        codes = torch.empty((self.P, cfg.H // 2), dtype=torch.uint8, device="cuda")
        sf = torch.empty((self.P // 128) * (cfg.H // 128) * 512, dtype=torch.uint8, device="cuda")
        M.moesq_quant_act(self.x.cuda().view(torch.uint16), cfg.H, st, eo, po, cfg.E, cuda(self.g_in_gu),
                          self.S, M.SF_KERNEL, codes, sf)
        return codes, sf


CASES = {
    "tiny": (W.CONFIGS["tiny"], 64),
    "ragged_multi_tile": (W.LayerConfig("ragged", 41, 4, 2, 384, 128, (400,), "uniform", True), 400),
    "sparse_routing": (W.LayerConfig("sparse", 43, 16, 1, 256, 256, (9,), "zipf", True), 9),
    "mid_ktail": (W.LayerConfig("mid", 42, 16, 4, 384, 256, (300,), "uniform", True), 300),
    # full 512-deep stages (one metadata copy per stage, 3-D token boxes), plus tiles of <= 32 tokens
    "deep_k": (W.LayerConfig("deep", 44, 12, 2, 1024, 512, (150,), "zipf", True), 150),
    # gate and up each scaled by its own global (no fold into the up block scales)
    "exact_per_half_alpha": (W.LayerConfig("exact", 45, 8, 2, 512, 256, (200,), "uniform", True), 200,
                             dict(exact=True)),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def layer(request):
    cfg, T, *opt = CASES[request.param]
    return Layer(cfg, T, **(opt[0] if opt else {}))


def test_gate_up_f32_within_tolerance(layer):
    L = layer
    eo, po, st, ts = L.device_routing()
    codes, sf = L.device_act(eo, po, st)
    out = torch.full((L.S, 2 * L.cfg.I), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moesq_grouped_gemm(L.dgu.struct, codes, sf, cuda(L.g_in_gu), eo, po, L.S, L.P, M.EPI_F32, None, out,
                         None, d_status=status)
    y = out.cpu().numpy().astype(np.float64)
    assert int(status.item()) == 0
    err = np.abs(y - L.acc_gu)
    lim = TOL * L.bound_gu + 1e-30
    assert np.isfinite(y).all()
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g} at {np.unravel_index(np.argmax(err / lim), err.shape)}"


def test_gate_up_bf16_within_tolerance(layer):
    """bf16 output of the gate_up GEMM: gate and up halves of a tile land in separate column ranges."""
    L = layer
    eo, po, st, ts = L.device_routing()
    codes, sf = L.device_act(eo, po, st)
    out = torch.full((L.S, 2 * L.cfg.I), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.moesq_grouped_gemm(L.dgu.struct, codes, sf, cuda(L.g_in_gu), eo, po, L.S, L.P, M.EPI_BF16, None,
                         out.view(torch.uint16), None)
    y = out.float().cpu().numpy().astype(np.float64)
    lim = TOL * L.bound_gu + bf16_ulp(L.acc_gu) + 1e-30
    assert np.isfinite(y).all()
    err = np.abs(y - L.acc_gu)
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"


def test_down_bf16_within_tolerance(layer):
    """down GEMM on NVFP4 activations quantised from a synthetic h (one row per slot)."""
    L = layer
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    rng = np.random.default_rng(3)
    h = F.bf16_round((rng.standard_normal((L.S, cfg.I)) * 2).astype(np.float32))
    g_in = L.g_in_dn
    e_of = R.slot_expert(L.perm["expert_offsets"])
    hc, hs = N.quantize_groups(h, g_in[e_of])
    Wd = [G.weight_int(s) for s in L.dn]
    yx, bound = G.grouped_gemm_exact(Wd, [s["g"][0] for s in L.dn], G.dequant_int(hc, hs), g_in,
                                     L.perm["expert_offsets"])
    codes = torch.empty((L.P, cfg.I // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((L.P // 128) * (cfg.I // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_quant_act(cuda(h, torch.bfloat16).view(torch.uint16), cfg.I, None, eo, po, cfg.E, cuda(g_in),
                      L.S, M.SF_KERNEL, codes, sf)
    y = torch.empty((L.S, cfg.H), dtype=torch.bfloat16, device="cuda")
    M.moesq_grouped_gemm(L.ddn.struct, codes, sf, cuda(g_in), eo, po, L.S, L.P, M.EPI_BF16, None,
                         y.view(torch.uint16), None)
    yg = y.float().cpu().numpy().astype(np.float64)
    lim = TOL * bound + bf16_ulp(yx) + 1e-30
    err = np.abs(yg - yx)
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"


def test_swiglu_requant_epilogue(layer):
    L = layer
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    codes, sf = L.device_act(eo, po, st)
    h_codes = torch.empty((L.P, cfg.I // 2), dtype=torch.uint8, device="cuda")
    h_sf = torch.empty((L.P // 128) * (cfg.I // 128) * 512, dtype=torch.uint8, device="cuda")
    M.moesq_grouped_gemm(L.dgu.struct, codes, sf, cuda(L.g_in_gu), eo, po, L.S, L.P, M.EPI_SWIGLU_NVFP4,
                         cuda(L.g_in_dn), h_codes, h_sf)
    got_c, got_s = PU.kernel_rows_to_slots(h_codes.cpu().numpy(), h_sf.cpu().numpy(),
                                           L.perm["expert_offsets"], L.perm["pad_offsets"], cfg.I)
    got_codes = N.unpack_codes(got_c)
    h = G.swiglu(L.acc_gu)
    e_of = R.slot_expert(L.perm["expert_offsets"])
    an = PU.requant_analysis(h, PU.swiglu_error_bound(L.acc_gu, L.bound_gu, TOL), L.g_in_dn[e_of])
    fixed = an["code_fixed"]
    assert np.array_equal(got_s[an["sc_fixed"]], an["sc"][an["sc_fixed"]])
    assert np.array_equal(got_codes[fixed], an["codes"][fixed])
    # the rest: a valid rounding -- dequantised value within the bracket of possible results
    g = L.g_in_dn[e_of].astype(np.float64)[:, None]
    deq_gpu = F.e2m1_decode(got_codes) * np.repeat(F.e4m3_decode(got_s), 32, axis=1) * g
    deq_ref = F.e2m1_decode(an["codes"]) * np.repeat(F.e4m3_decode(an["sc"]), 32, axis=1) * g
    assert (np.abs(deq_gpu - deq_ref) <= an["max_dev"] * (1 + 1e-6) + 1e-30).all()
    assert fixed.mean() > 0.95                  # the error bound is conservative; most codes are pinned


def test_moe_forward_end_to_end(layer):
    L = layer
    cfg = L.cfg
    ref = G.moe_forward(L.x.float().numpy(), L.ids, L.w, L.gu, L.dn, L.g_in_gu, L.g_in_dn, cfg.E, fold=not L.exact)
    moe = M.MoELayer(cfg.k, L.dgu, L.ddn, cuda(L.g_in_gu), cuda(L.g_in_dn))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.forward(L.x.cuda(), cuda(L.ids.astype(np.int32)), cuda(L.w), d_status=status)
    got = out.float().cpu().numpy().astype(np.float64)
    assert int(status.item()) == 0
    # bound: down tolerance + bf16 rounding of y + requant flips of h + the final bf16 rounding
    lim = PU.forward_error_limit(ref, L.dn, L.g_in_dn, L.w, TOL)
    err = np.abs(got - ref["out"])
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"
    # and the typical agreement is tight
    rel = np.linalg.norm(got - ref["out"]) / np.linalg.norm(ref["out"])
    assert rel < 2e-2


def test_moe_forward_host_matches_device(layer):
    L = layer
    cfg = L.cfg
    moe = M.MoELayer(cfg.k, L.dgu, L.ddn, cuda(L.g_in_gu), cuda(L.g_in_dn))
    dev_out = moe.forward(L.x.cuda(), cuda(L.ids.astype(np.int32)), cuda(L.w))
    h_out = torch.empty((L.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    moe.forward_host(L.x.pin_memory(), torch.from_numpy(L.ids.astype(np.int32)).pin_memory(),
                     torch.from_numpy(L.w).pin_memory(), h_out)
    assert torch.equal(h_out, dev_out.cpu())


def test_forward_is_deterministic(layer):
    L = layer
    cfg = L.cfg
    moe = M.MoELayer(cfg.k, L.dgu, L.ddn, cuda(L.g_in_gu), cuda(L.g_in_dn))
    a = moe.forward(L.x.cuda(), cuda(L.ids.astype(np.int32)), cuda(L.w))
    b = moe.forward(L.x.cuda(), cuda(L.ids.astype(np.int32)), cuda(L.w))
    assert torch.equal(a, b)
