"""GPU parity at the full sizes of the layer shapes the benchmark measures, in the
benchmark's own launch configuration (the staged pipeline of bench.py: weights
exported and repacked by the library, CTA-pair GEMMs, fused SwiGLU + NVFP4
requant), checked on sampled outputs the oracle computes one by one.

Per shape:

- the whole routing permutation is bit-exact;
- for the routed slots of one expert (the median-loaded one), these match the oracle:
  - the activation codes and scales, bit-exact;
  - the requantised SwiGLU codes and scales, bit-exact wherever the NVFP4 rule fixes them
    under the gate_up tolerance, a valid rounding elsewhere;
  - the bf16 down outputs y, within 1e-5 * sum|a w| plus the effect of those
    requantisation flips plus one bf16 ulp.

The oracle's inputs are the seeded generator's bf16 tensors (expert weights, layer input,
routing), drawn on the device and copied back.  The down-input global of the layer is a
value derived from the oracle's own SwiGLU output, never from a GPU result.
"""
import numpy as np
import pytest
import torch

import bench
import workloads as W
from oracle import formats as F
from oracle import gemm as G
from oracle import nvfp4 as N
from oracle import routing as R
from oracle import storage as S
from tests import parity_util as PU

pytestmark = pytest.mark.gpu

TOL = 1e-5
SLOTS = 6
FULL = [("qwen3_30b_a3b", 16384), ("qwen3_5_397b_a17b", 32768), ("qwen3_235b_a22b", 65536),
        ("kimi_k2", 16384)]


def bf16_ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def sf_of_rows(sf_blocks, rows, K):
    """Per-row [len(rows), K/32] scales out of the 512-byte block layout."""
    sfb = np.asarray(sf_blocks).reshape(-1, K // 128, 512)
    out = np.empty((rows.size, K // 32), np.uint8)
    r = rows % 128
    for g in range(K // 32):
        out[:, g] = sfb[rows // 128, g // 4, (r % 32) * 16 + (r // 32) * 4 + g % 4]
    return out


@pytest.mark.parametrize("name,T", FULL)
def test_full_size_sampled_parity(name, T):
    cfg = W.CONFIGS[name]
    dev = torch.device("cuda", 0)
    b = bench.Bench(cfg, T, dev)
    E, H, I = cfg.E, cfg.H, cfg.I

    # ---- oracle side: routing, one expert's slots, exact gate_up and SwiGLU
    ids = b.ids.cpu().numpy()
    ref = R.permute(ids, E)
    off = ref["expert_offsets"]
    counts = np.diff(off)
    nz = np.flatnonzero(counts)
    e = int(nz[np.argsort(counts[nz], kind="stable")[nz.size // 2]])
    n_e = int(counts[e])
    slots = np.unique(np.linspace(off[e], off[e + 1] - 1, min(SLOTS, n_e)).astype(np.int64))
    tokens = ref["slot_token"][slots]
    x_rows = b.x[torch.as_tensor(tokens, device=dev)].float().cpu().numpy()
    g_in = np.float32(W.activation_global_scale_input(b.x.cpu()))
    one = np.array([0, slots.size], np.int64)
    a_c, a_s = G.quant_act(x_rows, np.arange(slots.size), one, np.array([g_in], np.float32))
    n_seg = 2 if cfg.split_gate_up_global else 1
    st_gu = S.quantize_weight(W.expert_weights_bf16(cfg, e, "gate_up", dev).float().cpu().numpy(), n_seg)
    st_dn = S.quantize_weight(W.expert_weights_bf16(cfg, e, "down", dev).float().cpu().numpy(), 1)
    g_gu = np.asarray(st_gu["g"], np.float32).reshape(-1)
    sc = st_gu["scale"].copy()
    if g_gu.size == 2:
        sc[I:] = S.fold_up_scales(sc[I:], g_gu[0], g_gu[1])
    w_gu = G.dequant_int(N.unpack_codes(S.decode(st_gu["packed"], st_gu["mask"])), sc)
    acc, bound = G.grouped_gemm_exact([w_gu], [g_gu[0]], G.dequant_int(a_c, a_s), np.array([g_in]), one)
    h = G.swiglu(acc)
    g_dn = np.float32(np.float32(np.abs(h).max()) / np.float32(2688))   # from the oracle's h only

    # ---- GPU side: the benchmark's stages with that down-input global
    b.g_in_dn = torch.full((E,), float(g_dn), dtype=torch.float32, device=dev)
    for st in b.STAGES:
        getattr(b, st)()
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0

    assert np.array_equal(b.eo.cpu().numpy(), off)
    assert np.array_equal(b.po.cpu().numpy(), ref["pad_offsets"])
    assert np.array_equal(b.slot_token.cpu().numpy(), ref["slot_token"])
    assert np.array_equal(b.token_slot.cpu().numpy().reshape(T, cfg.k), ref["token_slot"])

    rows = R.padded_row_of_slot(off, ref["pad_offsets"])[slots]
    rows_t = torch.as_tensor(rows, device=dev)
    # activation codes and scales, bit-exact
    got_ac = b.a_codes[rows_t].cpu().numpy()
    want_ac = (a_c[:, 0::2] | (a_c[:, 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(got_ac, want_ac)
    assert np.array_equal(sf_of_rows(b.a_sf.cpu().numpy(), rows, H), a_s)

    # requantised SwiGLU output: pinned codes bit-exact, the rest a valid rounding
    got_hc = N.unpack_codes(b.h_codes[rows_t].cpu().numpy())
    got_hs = sf_of_rows(b.h_sf.cpu().numpy(), rows, I)
    an = PU.requant_analysis(h, PU.swiglu_error_bound(acc, bound, TOL), np.full(slots.size, g_dn, np.float32))
    fixed = an["code_fixed"]
    assert np.array_equal(got_hs[an["sc_fixed"]], an["sc"][an["sc_fixed"]])
    assert np.array_equal(got_hc[fixed], an["codes"][fixed])
    deq_gpu = F.e2m1_decode(got_hc) * np.repeat(F.e4m3_decode(got_hs), 32, axis=1) * np.float64(g_dn)
    deq_ref = F.e2m1_decode(an["codes"]) * np.repeat(F.e4m3_decode(an["sc"]), 32, axis=1) * np.float64(g_dn)
    assert (np.abs(deq_gpu - deq_ref) <= an["max_dev"] * (1 + 1e-6) + 1e-30).all()
    assert fixed.mean() > 0.95

    # down outputs y of the sampled slots: the oracle's own requantised h through the
    # exact down GEMM; the bound adds the tolerance, the flips' effect and one bf16 ulp
    w_dn = G.weight_int(st_dn)
    g_w_dn = np.float32(st_dn["g"][0])
    y_ref, bound_d = G.grouped_gemm_exact([w_dn], [g_w_dn], G.dequant_int(an["codes"], an["sc"]),
                                          np.array([g_dn]), one)
    flip = an["max_dev"] @ (np.abs(w_dn).astype(np.float64) * 2.0 ** -10 * np.float64(g_w_dn)).T
    y_gpu = b.y[torch.as_tensor(slots, device=dev)].float().cpu().numpy().astype(np.float64)
    lim = TOL * bound_d + flip + bf16_ulp(y_ref) + bf16_ulp(np.abs(y_ref) + flip) + 1e-30
    err = np.abs(y_gpu - y_ref)
    assert (err <= lim).all(), f"max err/lim {np.max(err / lim):.3g}"
    assert np.linalg.norm(y_gpu - y_ref) <= 2e-2 * np.linalg.norm(y_ref)
    del b
    torch.cuda.empty_cache()
