"""Expert parallelism's exchange logic on CPU ranks (gloo, rendezvous on 127.0.0.1).

Each rank holds a contiguous range of the experts and its own tokens; the dispatch
(NVFP4 codes and scales of every slot to the expert's rank) and the combine (bf16
outputs back, weighted sum on the token's rank) run through all_to_all_single.  The
per-rank compute here is the oracle (exact GEMMs, the NVFP4 rule, the j-order
combine), so the assembled result must equal the single-process oracle forward bit
for bit, whatever the split of experts and tokens.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    import workloads as W
    from oracle import gemm as G
    from oracle import routing as R
    from oracle import storage as S
    from tests import parity_util as PU
    cfg = W.LayerConfig("ep", 71, 8, 2, 256, 128, (48,), "uniform", True)
    T = 48
    gu = W.all_expert_weights_bf16(cfg, "gate_up")
    dn = W.all_expert_weights_bf16(cfg, "down")
    st_gu = [S.quantize_weight(gu[e].float().numpy(), 2) for e in range(cfg.E)]
    st_dn = [S.quantize_weight(dn[e].float().numpy(), 1) for e in range(cfg.E)]
    x = W.layer_input_bf16(cfg, T)
    ids, w = W.routing(cfg, T)
    g_in = np.full(cfg.E, W.activation_global_scale_input(x), np.float32)
    perm = R.permute(ids.numpy(), cfg.E)
    a_c, a_s = G.quant_act(x.float().numpy(), perm["slot_token"], perm["expert_offsets"], g_in)
    acc, _ = G.gate_up_exact(st_gu, G.dequant_int(a_c, a_s), g_in, perm["expert_offsets"])
    g_dn = PU.calibrate_g_in_down(acc, perm["expert_offsets"], cfg.E)
    return cfg, T, st_gu, st_dn, x, ids, w, g_in, g_dn


class OracleCompute:
    """The per-rank steps of sparse_nvfp4_moe_b200.ep with the oracle."""

    def __init__(self, st_gu, st_dn, g_in_all, g_dn_all, lo, hi, H):
        self.gu, self.dn = st_gu[lo:hi], st_dn[lo:hi]
        self.g_all, self.g_in_l, self.g_dn_l = g_in_all, g_in_all[lo:hi], g_dn_all[lo:hi]
        self.E_l, self.H = hi - lo, H

    def route(self, topk_ids, E):
        from oracle import routing as R
        p = R.permute(topk_ids.numpy(), E)
        return torch.from_numpy(p["expert_offsets"]), p["slot_token"], p["token_slot"]

    def quantise(self, x, slot_token, eo, E):
        from oracle import gemm as G
        from oracle import nvfp4 as N
        c, s = G.quant_act(x.float().numpy(), slot_token, eo.numpy(), self.g_all)
        return torch.from_numpy(N.pack_codes(c)), torch.from_numpy(s)

    def experts(self, codes, sf, local_ids):
        from oracle import formats as F
        from oracle import gemm as G
        from oracle import nvfp4 as N
        from oracle import routing as R
        n = codes.shape[0]
        if n == 0:
            return torch.empty((0, self.H), dtype=torch.bfloat16)
        A = G.dequant_int(N.unpack_codes(codes.numpy()), sf.numpy())
        p = R.permute(local_ids.numpy().reshape(n, 1), self.E_l)
        off, order = p["expert_offsets"], p["slot_token"]
        acc, _ = G.gate_up_exact(self.gu, A[order], self.g_in_l, off)
        h = G.swiglu(acc)
        e_of = R.slot_expert(off)
        hc, hs = N.quantize_groups(F.f32(h), self.g_dn_l[e_of])
        y, _ = G.grouped_gemm_exact([G.weight_int(s) for s in self.dn], [s["g"][0] for s in self.dn],
                                    G.dequant_int(hc, hs), self.g_dn_l, off)
        y_recv = np.empty_like(y)
        y_recv[order] = y
        return torch.from_numpy(F.bf16_round(F.f32(y_recv))).to(torch.bfloat16)

    def combine(self, y, token_slot, topk_w):
        from oracle import routing as R
        return torch.from_numpy(R.unpermute(y.float().numpy(), token_slot, topk_w.numpy())).to(torch.bfloat16)


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from sparse_nvfp4_moe_b200.ep import ExpertParallelMoE, expert_ranges
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        cfg, T, st_gu, st_dn, x, ids, w, g_in, g_dn = _layer()
        lo, hi = expert_ranges(cfg.E, world)[rank]
        t0, t1 = rank * T // world, (rank + 1) * T // world       # this rank's tokens
        ep = ExpertParallelMoE(cfg.E, cfg.k, cfg.H, OracleCompute(st_gu, st_dn, g_in, g_dn, lo, hi, cfg.H))
        out = ep.forward(x[t0:t1], ids[t0:t1], w[t0:t1])
        q.put((rank, t0, out.view(torch.int16).numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_equals_single_process(world):
    sys.path.insert(0, ROOT)
    from oracle import gemm as G
    cfg, T, st_gu, st_dn, x, ids, w, g_in, g_dn = _layer()
    ref = G.moe_forward(x.float().numpy(), ids.numpy(), w.numpy(), st_gu, st_dn, g_in, g_dn, cfg.E)
    want = torch.from_numpy(ref["y_bf16_combined"]).to(torch.bfloat16).view(torch.int16).numpy()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank, args=(world, _free_port(), q), nprocs=world, join=True, start_method="spawn")
    got = np.empty_like(want)
    for _ in range(world):
        r, t0, o = q.get()
        got[t0:t0 + o.shape[0]] = o
    assert np.array_equal(got, want)


def test_expert_ranges_cover_all_experts():
    sys.path.insert(0, ROOT)
    from sparse_nvfp4_moe_b200.ep import expert_ranges
    for E, G in ((8, 2), (8, 3), (384, 8), (5, 8)):
        r = expert_ranges(E, G)
        assert r[0][0] == 0 and r[-1][1] == E and all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert max(h - l for l, h in r) - min(h - l for l, h in r) <= 1
