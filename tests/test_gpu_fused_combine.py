"""The down GEMM with the weighted combine fused into its epilogue
(moesq_grouped_gemm_down_combine) against the two-kernel path it can replace and
against the oracle.

The fused path sums a token's k weighted rows of each 128-output tile in j order in
float32 without fused multiply-add, once all k slots of the token have arrived (an
arrival count per token and tile), so it must be bit-identical to the bf16 down GEMM
followed by moesq_unpermute.  Each case checks:

* every slot's y row bit-identical to the bf16 epilogue's;
* the combined output bit-identical to moesq_unpermute of that y;
* the combined output within the down-GEMM tolerance of the oracle's exact sum
  sum_j w_j * y_exact (1e-5 * sum|a w| per slot row, one bf16 ulp of each stored y row,
  one bf16 ulp of the output), independently of the two-kernel path.

Cases: the layers of tests/test_gpu_gemm.py, a top-1 layer (every count completes at
its first arrival), the decode-sized layer of tests/test_gpu_multi_item.py (items from
the set-up table) and its 512-item layer, at the uncapped launch and on 1 and 3 CTA
pairs (one pair then produces many of a token's arrivals, in another order).  The
combine is the weighted sum of the MoESQ README's expert path; the grouped GEMM is the
kernel line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card.
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
from tests import test_gpu_gemm as TG
from tests import test_gpu_multi_item as TM
from tests.parity_util import cuda

pytestmark = pytest.mark.gpu

TOL = 1e-5
TOP1 = W.LayerConfig("combine_top1", 50, 8, 1, 512, 256, (300,), "uniform", True)
LAYERS = {name: TG.CASES[name] for name in TG.CASES}
LAYERS["top1"] = (TOP1, 300)
LAYERS["decode_items"] = (TM.DECODE, 256)
LAYERS["many_items"] = (TM.MANY, 8192)


@pytest.fixture(scope="module", params=sorted(LAYERS))
def layer(request):
    cfg, T, *opt = LAYERS[request.param]
    return TG.Layer(cfg, T, **(opt[0] if opt else {}))


def _down_inputs(L):
    """Routing, NVFP4 down input from a seeded synthetic h, and the oracle's exact y."""
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    rng = np.random.default_rng(5)
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
    return eo, po, st, ts, codes, sf, yx, bound


@pytest.mark.parametrize("limit", (0, 1, 3))
def test_fused_combine_matches_two_kernels_and_oracle(layer, limit):
    L = layer
    cfg = L.cfg
    eo, po, st, ts, codes, sf, yx, bound = _down_inputs(L)
    w = cuda(L.w)
    g_in = cuda(L.g_in_dn)
    with TM.PairLimit(limit):
        y_ref = torch.empty((L.S, cfg.H), dtype=torch.bfloat16, device="cuda")
        M.moesq_grouped_gemm(L.ddn.struct, codes, sf, g_in, eo, po, L.S, L.P, M.EPI_BF16, None,
                             y_ref.view(torch.uint16), None)
        out_ref = torch.empty((L.T, cfg.H), dtype=torch.bfloat16, device="cuda")
        M.moesq_unpermute(y_ref.view(torch.uint16), ts, w, L.T, cfg.k, cfg.H, out_ref.view(torch.uint16))

        y = torch.full((L.S, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        out = torch.full((L.T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        arrivals = torch.full((L.T * (cfg.H // 128),), 7, dtype=torch.int32, device="cuda")  # cleared by the call
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        M.moesq_grouped_gemm_down_combine(L.ddn.struct, codes, sf, g_in, eo, po, L.S, L.P, st, ts, w, L.T, cfg.k,
                                          y.view(torch.uint16), out.view(torch.uint16), arrivals, status)
        torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    assert bool((arrivals == cfg.k).all())  # every (token, tile) saw exactly k arrivals
    # the oracle: sum_j w_j y_exact over the token's slots, in float64
    slot = L.perm["token_slot"]                       # [T, k]
    wv = L.w.astype(np.float64)
    want = np.einsum("tj,tjh->th", wv, yx[slot])
    ulp = TG.bf16_ulp
    lim_rows = TOL * bound + ulp(yx) + 1e-30          # per slot row, as the down GEMM test
    lim = np.einsum("tj,tjh->th", np.abs(wv), lim_rows[slot])
    lim = lim + ulp(np.abs(want) + lim) + 1e-30
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - want)
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"


def test_fused_combine_arguments():
    L = TG.Layer(*TG.CASES["tiny"])
    cfg = L.cfg
    eo, po, st, ts = L.device_routing()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    y = torch.empty((L.S, cfg.H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((L.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    arr = torch.zeros(L.T * (cfg.H // 128), dtype=torch.int32, device="cuda")
    codes = torch.zeros((L.P, cfg.I // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((L.P // 128) * (cfg.I // 128) * 512, dtype=torch.uint8, device="cuda")
    g = cuda(L.g_in_dn)
    w = cuda(L.w)
    with pytest.raises(M.MoesqError):   # S != T * k
        M.moesq_grouped_gemm_down_combine(L.ddn.struct, codes, sf, g, eo, po, L.S, L.P, st, ts, w, L.T + 1,
                                          cfg.k, y.view(torch.uint16), out.view(torch.uint16), arr)
    with pytest.raises(M.MoesqError):   # gate_up weights
        M.moesq_grouped_gemm_down_combine(L.dgu.struct, codes, sf, g, eo, po, L.S, L.P, st, ts, w, L.T, cfg.k,
                                          y.view(torch.uint16), out.view(torch.uint16), arr)
    with pytest.raises(M.MoesqError):   # missing routing
        M.moesq_grouped_gemm_down_combine(L.ddn.struct, codes, sf, g, eo, po, L.S, L.P, None, ts, w, L.T, cfg.k,
                                          y.view(torch.uint16), out.view(torch.uint16), arr)
    del dummy
