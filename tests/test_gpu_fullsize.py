"""GPU parity at the full sizes of the layer shapes the benchmark measures, in the
benchmark's own launch configuration (the staged pipeline of bench.py: weights
exported and repacked by the library, CTA-pair GEMMs, fused SwiGLU + NVFP4
requant, weighted combine), checked on samples the oracle computes one by one.

Per shape:

- the whole routing permutation is bit-exact;
- sampled slots of these experts are checked against the oracle:
  - the 4 largest non-empty experts (at Qwen3.5-397B-A17B, T = 32768 one of them holds
    about 32 k tokens): every one of their token tiles, 8 slots of each (the first two,
    the last two and four seeded random ones), so every work item the persistent
    schedule runs on a giant group is sampled at both tile edges;
  - the 4 smallest non-empty experts, 2 seeded random experts, and every expert of 2
    seeded random tokens: all their slots (tiles sampled as above where an expert holds
    more than 1024);
  checks: the activation codes and scales bit-exact; the requantised SwiGLU codes and
  scales bit-exact wherever the NVFP4 rule fixes them under the gate_up tolerance and
  a valid rounding elsewhere; the bf16 down outputs y within 1e-5 * sum|a w| plus the
  effect of those requantisation flips plus one bf16 ulp;
- the combined output rows of the 2 random tokens (all k of their slots computed by
  the oracle end to end) within the same per-element forward bound as the small tests.

The oracle's inputs are the seeded generator's bf16 tensors (expert weights, layer
input, routing), drawn on the device and copied back; the oracle exports each expert's
storage itself (a spawned process pool spreads that over the host cores).  The down
input global of the layer is derived from the oracle's own SwiGLU outputs, never from a
GPU result.  The grouped GEMM is the kernel line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ
model card; the layer shapes follow the "Supported models" table of the MoESQ README.
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
from tests import oracle_pool
from tests import parity_util as PU

pytestmark = pytest.mark.gpu

TOL = 1e-5
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


def bits(t):
    """bf16 device tensor -> its 16-bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def tile_sample(n, rng):
    """Slots (0..n-1 of one expert) sampled per 128-slot token tile: the first two, the
    last two and four random ones of every tile."""
    out = []
    for q0 in range(0, n, 128):
        q1 = min(n, q0 + 128)
        edge = [q0, q0 + 1, q1 - 2, q1 - 1]
        mid = rng.choice(np.arange(q0, q1), size=min(4, q1 - q0), replace=False)
        out.append(np.concatenate([edge, mid]))
    return np.unique(np.clip(np.concatenate(out), 0, n - 1)) if out else np.zeros(0, np.int64)


@pytest.mark.timeout(1200)
@pytest.mark.parametrize("name,T", FULL)
def test_full_size_sampled_parity(name, T):
    cfg = W.CONFIGS[name]
    dev = torch.device("cuda", 0)
    b = bench.Bench(cfg, T, dev)
    E, H, I, k = cfg.E, cfg.H, cfg.I, cfg.k
    rng = np.random.default_rng(7)

    # ---- which slots: the oracle's own routing permutation
    ids = b.ids.cpu().numpy()
    ref = R.permute(ids, E)
    off = ref["expert_offsets"]
    counts = np.diff(off)
    nz = np.flatnonzero(counts)
    by_size = nz[np.argsort(counts[nz], kind="stable")]
    large, small = [int(e) for e in by_size[-4:]], [int(e) for e in by_size[:4]]
    others = [int(e) for e in nz if e not in large + small]
    rand_e = [int(e) for e in rng.choice(others, size=min(2, len(others)), replace=False)]
    comb_tokens = np.sort(rng.choice(T, size=2, replace=False))
    comb_slots = ref["token_slot"][comb_tokens].reshape(-1)
    comb_e = set(int(e) for e in ids[comb_tokens].reshape(-1))
    experts = sorted(set(large) | set(small) | set(rand_e) | comb_e)
    slots = {}
    for e in experts:
        n = int(counts[e])
        local = tile_sample(n, rng) if (e in large or n > 1024) else np.arange(n)
        sl = set((off[e] + local).tolist())
        sl |= set(int(s) for s in comb_slots if off[e] <= s < off[e + 1])
        slots[e] = np.array(sorted(sl), np.int64)
        # every 128-slot token tile of the expert is sampled
        assert set(((slots[e] - off[e]) // 128).tolist()) == set(range(-(-n // 128)))
    all_slots = np.concatenate([slots[e] for e in experts])

    # ---- oracle: storages of every sampled expert, activations, exact gate_up and SwiGLU
    n_seg = 2 if cfg.split_gate_up_global else 1
    tasks = [(e, bits(W.expert_weights_bf16(cfg, e, "gate_up", dev)), bits(W.expert_weights_bf16(cfg, e, "down", dev)),
              n_seg) for e in experts]
    st = oracle_pool.export_experts(tasks)
    del tasks
    g_in = np.float32(W.activation_global_scale_input(b.x.cpu()))
    tokens = ref["slot_token"][all_slots]
    x_rows = b.x[torch.as_tensor(tokens, device=dev)].float().cpu().numpy()
    a_c_all, a_s_all = G.quant_act(x_rows, np.arange(all_slots.size), np.array([0, all_slots.size]),
                                   np.array([g_in], np.float32))
    pos = {int(s): i for i, s in enumerate(all_slots)}
    per = {}
    for e in experts:
        idx = np.array([pos[int(s)] for s in slots[e]], np.int64)
        gu, dn = st[e]
        g_gu = np.asarray(gu["g"], np.float32).reshape(-1)
        sc = gu["scale"].copy()
        if g_gu.size == 2:
            sc[I:] = S.fold_up_scales(sc[I:], g_gu[0], g_gu[1])
        w_gu = G.dequant_int(N.unpack_codes(S.decode(gu["packed"], gu["mask"])), sc)
        one = np.array([0, idx.size], np.int64)
        acc, bound = G.grouped_gemm_exact([w_gu], [g_gu[0]], G.dequant_int(a_c_all[idx], a_s_all[idx]),
                                          np.array([g_in]), one)
        per[e] = dict(idx=idx, acc=acc, bound=bound, h=G.swiglu(acc))
    h_max = max(float(np.abs(v["h"]).max()) for v in per.values())
    g_dn = np.float32(np.float32(h_max) / np.float32(2688))   # from the oracle's h only

    # ---- GPU side: the benchmark's stages with that down-input global
    b.g_in_dn = torch.full((E,), float(g_dn), dtype=torch.float32, device=dev)
    for s_ in b.STAGES:
        getattr(b, s_)()
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0

    assert np.array_equal(b.eo.cpu().numpy(), off)
    assert np.array_equal(b.po.cpu().numpy(), ref["pad_offsets"])
    assert np.array_equal(b.slot_token.cpu().numpy(), ref["slot_token"])
    assert np.array_equal(b.token_slot.cpu().numpy().reshape(T, k), ref["token_slot"])

    prow_all = R.padded_row_of_slot(off, ref["pad_offsets"])
    a_sf_host, h_sf_host = b.a_sf.cpu().numpy(), b.h_sf.cpu().numpy()
    y_lim, y_ref = {}, {}
    comb_set = set(int(x) for x in comb_slots)
    for e in experts:
        v = per[e]
        sl, idx = slots[e], v["idx"]
        rows = prow_all[sl]
        rows_t = torch.as_tensor(rows, device=dev)
        # activation codes and scales, bit-exact
        a_c, a_s = a_c_all[idx], a_s_all[idx]
        assert np.array_equal(b.a_codes[rows_t].cpu().numpy(), (a_c[:, 0::2] | (a_c[:, 1::2] << 4)).astype(np.uint8)), e
        assert np.array_equal(sf_of_rows(a_sf_host, rows, H), a_s), e
        # requantised SwiGLU output: pinned codes bit-exact, the rest a valid rounding
        got_hc = N.unpack_codes(b.h_codes[rows_t].cpu().numpy())
        got_hs = sf_of_rows(h_sf_host, rows, I)
        an = PU.requant_analysis(v["h"], PU.swiglu_error_bound(v["acc"], v["bound"], TOL),
                                 np.full(sl.size, g_dn, np.float32))
        fixed = an["code_fixed"]
        assert np.array_equal(got_hs[an["sc_fixed"]], an["sc"][an["sc_fixed"]]), e
        assert np.array_equal(got_hc[fixed], an["codes"][fixed]), e
        deq_gpu = F.e2m1_decode(got_hc) * np.repeat(F.e4m3_decode(got_hs), 32, axis=1) * np.float64(g_dn)
        deq_ref = F.e2m1_decode(an["codes"]) * np.repeat(F.e4m3_decode(an["sc"]), 32, axis=1) * np.float64(g_dn)
        assert (np.abs(deq_gpu - deq_ref) <= an["max_dev"] * (1 + 1e-6) + 1e-30).all(), e
        assert fixed.mean() > 0.95
        # down outputs y: the oracle's own requantised h through the exact down GEMM
        dn = st[e][1]
        w_dn = G.weight_int(dn)
        g_w_dn = np.float32(dn["g"][0])
        one = np.array([0, sl.size], np.int64)
        yr, bound_d = G.grouped_gemm_exact([w_dn], [g_w_dn], G.dequant_int(an["codes"], an["sc"]), np.array([g_dn]),
                                           one)
        flip = an["max_dev"] @ (np.abs(w_dn).astype(np.float64) * 2.0 ** -10 * np.float64(g_w_dn)).T
        lim = TOL * bound_d + flip + bf16_ulp(yr) + bf16_ulp(np.abs(yr) + flip) + 1e-30
        y_gpu = b.y[torch.as_tensor(sl, device=dev)].float().cpu().numpy().astype(np.float64)
        err = np.abs(y_gpu - yr)
        assert (err <= lim).all(), f"expert {e}: max err/lim {np.max(err / lim):.3g}"
        assert np.linalg.norm(y_gpu - yr) <= 2e-2 * np.linalg.norm(yr)
        for i, s_ in enumerate(sl):
            if s_ in comb_set:
                y_lim[int(s_)], y_ref[int(s_)] = lim[i], yr[i]

    # ---- the combined rows of the sampled tokens, every slot computed by the oracle
    w = b.w.cpu().numpy()
    out_gpu = b.out[torch.as_tensor(comb_tokens, device=dev)].float().cpu().numpy().astype(np.float64)
    for i, t in enumerate(comb_tokens):
        ts = ref["token_slot"][t]
        want = sum(np.float64(w[t, j]) * y_ref[int(ts[j])] for j in range(k))
        lim = sum(np.abs(np.float64(w[t, j])) * y_lim[int(ts[j])] for j in range(k))
        lim = lim + bf16_ulp(np.abs(want) + lim) + 1e-30
        assert (np.abs(out_gpu[i] - want) <= lim).all(), f"token {t}: max err/lim {np.max(np.abs(out_gpu[i] - want) / lim):.3g}"
    del b
    torch.cuda.empty_cache()
