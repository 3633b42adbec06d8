#!/usr/bin/env python
"""Benchmark of the paired-4:8 sparse NVFP4 MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config qwen3_30b_a3b] [--tokens T] [--no-sweep]

A step is one pass of the whole routed-expert path over one synthetic batch:
permute -> NVFP4 activation quantisation -> gate_up sparse grouped GEMM with the
fused SwiGLU + NVFP4 requant epilogue -> down sparse grouped GEMM -> weighted
combine.  Weights are drawn (bf16 N(0, 0.02)), pruned, quantised and encoded to
pair-bitmask storage by the library's own kernels, then repacked.  Inputs sit
in HBM before timing; L2 is flushed (a 256 MiB write) between timed steps and
every stage is timed with CUDA events on the launch stream.

Metric: dense-equivalent TFLOP/s (2*S*2I*H + 2*S*H*I per step, S = tokens*k),
whole job over all ranks.  Multi-GPU runs are replicas (weak scaling): every
rank runs the same layer on its own batch, no collective on the data path.

--impl reference times the CPU oracle (numpy, float64/int64) on a bounded sample
of the same workload on the host cores; it is a deliberately slow program.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dense-equiv TFLOP/s & % roofline, sparse NVFP4 MoE grouped GEMM (1 B200)"
UNIT = "TFLOP/s"
B_W, B_A = 0.34375, 0.53125     # bytes per dense element: sparse weight storage, NVFP4-32 activation
FP4_SPARSE_OVER_BF16 = 8.0      # nominal dense-equivalent sparse FP4 (18 PF) / dense bf16 (2.25 PF)
KERNELS_PER_STEP = 7            # permute x3, routed quant, gate_up GEMM, down GEMM, combine


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="qwen3_30b_a3b")
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-slots", type=int, default=2048, help="slots in the CPU-baseline sample")
    ap.add_argument("--storage", action="store_true",
                    help="storage benchmark instead: decode / re-encode / repack every expert's "
                         "pair-bitmask tensors of --config (default kimi_k2 with this flag)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def step_flops(S, H, I):
    return dict(gate_up=2.0 * S * 2 * I * H, down=2.0 * S * H * I)


def step_bytes(S, T, H, I, n_touched):
    return dict(
        gate_up=n_touched * 2 * I * H * B_W + S * H * B_A + S * I * B_A,
        down=n_touched * H * I * B_W + S * I * B_A + S * H * 2,
        quant_act=T * H * 2 + S * H * B_A,
        combine=S * H * 2 + T * H * 2,
        permute=S * 4 * 4,
    )


# --------------------------------------------------------------- clocks -----
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ our arm -------
class Bench:
    def __init__(self, cfg, T, device, lin=None):
        import numpy as np
        import torch

        import sparse_nvfp4_moe_b200 as M
        import workloads as W
        self.np, self.torch, self.M, self.W = np, torch, M, W
        self.cfg, self.T, self.dev = cfg, T, device
        n_seg = 2 if cfg.split_gate_up_global else 1
        kind = M.KIND_GATE_UP_SPLIT if n_seg == 2 else M.KIND_GATE_UP
        # weights: drawn on the device, exported and repacked by the library
        self.lin = lin if lin is not None else {}
        for which, ns, kd in (("gate_up", n_seg, kind), ("down", 1, M.KIND_DOWN)):
            if which in self.lin:
                continue
            w = W.all_expert_weights_bf16(cfg, which, device=device)
            st = M.quantize_expert_weights(w, ns)
            del w
            self.lin[which] = M.ExpertLinear.from_storage(st, kd)
            del st
        torch.cuda.empty_cache()
        self.x = W.layer_input_bf16(cfg, T, device=device)
        ids, w = W.routing(cfg, T, device=device)
        self.ids, self.w = ids.contiguous(), w.contiguous()
        self.S = T * cfg.k
        self.P = M.padded_rows(self.S, cfg.E)
        E = cfg.E
        i32 = dict(dtype=torch.int32, device=device)
        self.eo = torch.empty(E + 1, **i32)
        self.po = torch.empty(E + 1, **i32)
        self.slot_token = torch.empty(self.S, **i32)
        self.token_slot = torch.empty(self.S, **i32)
        self.perm_ws_n = M.permute_workspace_size(T, cfg.k, E)
        self.perm_ws = torch.empty(max(self.perm_ws_n, 16), dtype=torch.uint8, device=device)
        u8 = dict(dtype=torch.uint8, device=device)
        H, I = cfg.H, cfg.I
        self.a_codes = torch.empty((self.P, H // 2), **u8)
        self.a_sf = torch.empty((self.P // 128) * (H // 128) * 512, **u8)
        self.h_codes = torch.empty((self.P, I // 2), **u8)
        self.h_sf = torch.empty((self.P // 128) * (I // 128) * 512, **u8)
        self.y = torch.empty((self.S, H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.g_in_gu = torch.full((E,), W.activation_global_scale_input(self.x), dtype=torch.float32,
                                  device=device)
        self.g_in_dn = self.calibrate_down_globals()
        self.layer = M.MoELayer(cfg.k, self.lin["gate_up"], self.lin["down"], self.g_in_gu, self.g_in_dn)
        counts = torch.diff(self.eo.long()).cpu()
        self.n_touched = int((counts > 0).sum())
        self.max_group = int(counts.max())

    def calibrate_down_globals(self):
        """Static down-input globals: amax of silu(gate)*up per expert / (6*448), from one
        FP32-epilogue pass of the library's gate_up GEMM (set-up only, not timed)."""
        torch, M = self.torch, self.M
        self.permute()
        self.quant_act()
        acc = torch.empty((self.S, 2 * self.cfg.I), dtype=torch.float32, device=self.dev)
        M.moesq_grouped_gemm(self.lin["gate_up"].struct, self.a_codes, self.a_sf, self.g_in_gu, self.eo,
                             self.po, self.S, self.P, M.EPI_F32, None, acc, None, d_status=self.status)
        I = self.cfg.I
        h = torch.nn.functional.silu(acc[:, :I]) * acc[:, I:]
        amax_slot = h.abs().amax(dim=1)
        del acc, h
        eo = self.eo.long()
        e_of = torch.repeat_interleave(torch.arange(self.cfg.E, device=self.dev), torch.diff(eo))
        amax = torch.zeros(self.cfg.E, device=self.dev).scatter_reduce(0, e_of, amax_slot, "amax")
        g = amax / 2688.0
        nz = g[g > 0]
        g[g == 0] = nz.median() if nz.numel() else 1e-3
        return g.float().contiguous()

    # ---- the stages of one step, each a C-ABI call
    def permute(self):
        self.M.moesq_permute(self.ids, self.T, self.cfg.k, self.cfg.E, self.eo, self.po, self.slot_token,
                             self.token_slot, self.perm_ws, self.perm_ws_n, self.status)

    def quant_act(self):
        self.M.moesq_quant_act_routed(self.x.view(self.torch.uint16), self.T, self.cfg.H, self.ids,
                                      self.token_slot, self.cfg.k, self.eo, self.po, self.cfg.E, self.g_in_gu,
                                      self.a_codes, self.a_sf)

    def gemm_gate_up(self):
        self.M.moesq_grouped_gemm(self.lin["gate_up"].struct, self.a_codes, self.a_sf, self.g_in_gu, self.eo,
                                  self.po, self.S, self.P, self.M.EPI_SWIGLU_NVFP4, self.g_in_dn,
                                  self.h_codes, self.h_sf, d_status=self.status)

    def gemm_down(self):
        self.M.moesq_grouped_gemm(self.lin["down"].struct, self.h_codes, self.h_sf, self.g_in_dn, self.eo,
                                  self.po, self.S, self.P, self.M.EPI_BF16, None, self.y.view(self.torch.uint16),
                                  None, d_status=self.status)

    def combine(self):
        self.M.moesq_unpermute(self.y.view(self.torch.uint16), self.token_slot, self.w, self.T, self.cfg.k,
                               self.cfg.H, self.out.view(self.torch.uint16))

    STAGES = ("permute", "quant_act", "gemm_gate_up", "gemm_down", "combine")

    def graphs(self):
        """The step as one CUDA graph, and each stage as its own graph (for the
        per-kernel breakdown).  Replays carry no host launch gaps inside a graph."""
        torch = self.torch
        if getattr(self, "_graphs", None) is None:
            for s in self.STAGES:       # first calls outside capture (one-time attribute set-up)
                getattr(self, s)()
            torch.cuda.synchronize()
            self._graphs = {}
            for s in self.STAGES:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    getattr(self, s)()
                self._graphs[s] = g
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for s in self.STAGES:
                    getattr(self, s)()
            self._graphs["step"] = g
            torch.cuda.synchronize()
        return self._graphs

    def run(self, steps, warmup, flush):
        """Whole-step times (one graph per step) and per-stage times (one graph per
        stage), each step after an L2 flush and a GPU sleep that keeps the host ahead."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        graphs = self.graphs()
        for _ in range(warmup):
            graphs["step"].replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.nvtx.range_push("timed")
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            torch.cuda._sleep(1_000_000)
            ev[i][0].record(stream)
            graphs["step"].replay()
            ev[i][1].record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in self.STAGES] for _ in range(steps)]
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            torch.cuda._sleep(1_000_000)
            for j, s in enumerate(self.STAGES):
                evs[i][j][0].record(stream)
                graphs[s].replay()
                evs[i][j][1].record(stream)
        torch.cuda.synchronize()
        per = {s: [evs[i][j][0].elapsed_time(evs[i][j][1]) for i in range(steps)] for j, s in enumerate(self.STAGES)}
        return step_ms, per

    def dense_comparison(self, steps, flush):
        """The same two GEMMs with the dense comparison kernel on the decoded weights (the
        pages' --no-sparse-storage form): the seeded weights are exported again (the same
        bytes as the sparse layer's), decoded, and the scale blocks expanded to 16
        elements.  Timed like the stages of run(); the 16-element expansion of the
        activation scales is outside the timed GEMMs."""
        torch, M, W, cfg = self.torch, self.M, self.W, self.cfg
        dev = self.dev

        def expand(sf):
            o = torch.empty(sf.numel() * 2, dtype=torch.uint8, device=dev)
            M.moesq_sf_expand_block16(sf, o, sf.numel() // 512)
            return o

        dense = {}
        for which, ns in (("gate_up", 2 if cfg.split_gate_up_global else 1), ("down", 1)):
            lin = self.lin[which]
            w = W.all_expert_weights_bf16(cfg, which, device=dev)
            st = M.quantize_expert_weights(w, ns)
            del w
            codes = torch.empty((lin.E, lin.out, lin.K // 2), dtype=torch.uint8, device=dev)
            M.moesq_decode(st["packed"], st["mask"], codes, lin.E * lin.out, lin.K, self.status)
            assert torch.equal(st["packed"], lin.packed), "re-export differs from the sparse layer's weights"
            del st
            sf16 = expand(lin.sf)
            dense[which] = (codes, sf16, M.Linear(codes.data_ptr(), 0, sf16.data_ptr(), lin.alpha_w.data_ptr(),
                                                  lin.out, lin.K, lin.E, lin.kind))
        torch.cuda.empty_cache()
        self.permute()
        self.quant_act()
        a_sf16 = expand(self.a_sf)
        h_codes = torch.empty_like(self.h_codes)
        h_sf = torch.empty_like(self.h_sf)
        y = torch.empty_like(self.y)
        h_sf16 = torch.empty(h_sf.numel() * 2, dtype=torch.uint8, device=dev)

        def gate_up():
            M.moesq_grouped_gemm_dense(dense["gate_up"][2], self.a_codes, a_sf16, self.g_in_gu, self.eo, self.po,
                                       self.S, self.P, M.EPI_SWIGLU_NVFP4, self.g_in_dn, h_codes, h_sf,
                                       d_status=self.status)

        def down():
            M.moesq_grouped_gemm_dense(dense["down"][2], h_codes, h_sf16, self.g_in_dn, self.eo, self.po, self.S,
                                       self.P, M.EPI_BF16, None, y.view(torch.uint16), None, d_status=self.status)

        gate_up()
        M.moesq_sf_expand_block16(h_sf, h_sf16, h_sf.numel() // 512)
        down()
        torch.cuda.synchronize()
        graphs = {}
        for name, fn in (("gate_up", gate_up), ("down", down)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs[name] = g
        stream = torch.cuda.current_stream()
        res = {}
        for name, g in graphs.items():
            for _ in range(3):
                g.replay()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for a, b in ev:
                if flush is not None:
                    flush.zero_()
                torch.cuda._sleep(1_000_000)
                a.record(stream)
                g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            res[name] = sum(a.elapsed_time(b) for a, b in ev) / steps
        del graphs
        return res

    def check_against_forward(self):
        """The staged step and the single moesq_moe_forward call give identical bytes."""
        torch = self.torch
        for s in self.STAGES:
            getattr(self, s)()
        ref = self.out.clone()
        got = self.layer.forward(self.x, self.ids, self.w)
        torch.cuda.synchronize()
        return bool(torch.equal(ref, got))

    def e2e(self, steps, warmup):
        """Same metric through the host-buffer C-ABI call (H2D + layer + D2H, synchronised)."""
        torch = self.torch
        hx = self.x.cpu().pin_memory()
        hids = self.ids.cpu().pin_memory()
        hw = self.w.cpu().pin_memory()
        hout = torch.empty((self.T, self.cfg.H), dtype=torch.bfloat16).pin_memory()
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            self.layer.forward_host(hx, hids, hw, hout)
        times = []
        for _ in range(steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            self.layer.forward_host(hx, hids, hw, hout)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        h2d = hx.numel() * 2 + hids.numel() * 4 + hw.numel() * 4
        d2h = hout.numel() * 2
        return sum(times) / len(times), h2d, d2h


def cpu_baseline(cfg, T, n_slots, device_ids=None):
    """The oracle as it stands, on a bounded sample: the most-loaded expert's MLP
    (quantise -> exact gate_up -> SwiGLU -> requant -> exact down) for n routed slots."""
    import numpy as np
    import torch

    import workloads as W
    from oracle import gemm as G
    from oracle import nvfp4 as N
    from oracle import routing as R
    from oracle import storage as S

    ids, _ = W.routing(cfg, T) if device_ids is None else (device_ids, None)
    ids = np.asarray(ids)
    perm = R.permute(ids, cfg.E)
    counts = np.diff(perm["expert_offsets"])
    e = int(np.argmax(counts))
    n = int(min(n_slots, counts[e]))
    rows = perm["slot_token"][perm["expert_offsets"][e]:perm["expert_offsets"][e] + n]
    x = W.layer_input_bf16(cfg, T).float().numpy()[rows]
    n_seg = 2 if cfg.split_gate_up_global else 1
    t0 = time.perf_counter()
    gu = S.quantize_weight(W.expert_weights_bf16(cfg, e, "gate_up").float().numpy(), n_seg)
    dn = S.quantize_weight(W.expert_weights_bf16(cfg, e, "down").float().numpy(), 1)
    t_prep = time.perf_counter() - t0
    g_in = np.float32(np.abs(x).max() / 2688.0)
    t0 = time.perf_counter()
    ac, asf = N.quantize_groups(x, g_in)
    sc = gu["scale"].copy()
    if n_seg == 2:
        sc[cfg.I:] = S.fold_up_scales(sc[cfg.I:], gu["g"][0], gu["g"][1])
    Wg = G.dequant_int(N.unpack_codes(S.decode(gu["packed"], gu["mask"])), sc)
    acc, _ = G.grouped_gemm_exact([Wg], [gu["g"][0]], G.dequant_int(ac, asf), np.float32([g_in]),
                                  np.array([0, n]))
    h = G.swiglu(acc)
    g_dn = np.float32(np.abs(h).max() / 2688.0)
    hc, hs = N.quantize_groups(h.astype(np.float32), g_dn)
    G.grouped_gemm_exact([G.weight_int(dn)], [dn["g"][0]], G.dequant_int(hc, hs), np.float32([g_dn]),
                         np.array([0, n]))
    dt = time.perf_counter() - t0
    flops = 2.0 * n * (2 * cfg.I * cfg.H + cfg.H * cfg.I)
    return dict(value=flops / dt / 1e12, unit=UNIT, cores=1, kind="oracle",
                sample=(f"expert {e} ({counts[e]} routed slots) of the {cfg.name}-shaped layer at T={T}: "
                        f"quantise, exact int64 gate_up, SwiGLU, requant, exact int64 down for {n} slots "
                        f"({flops / 1e9:.1f} dense-equiv GFLOP in {dt:.1f} s; numpy int64 matmul is "
                        f"single-threaded; weight export {t_prep:.1f} s excluded)"),
                seconds=dt)


def traffic_record():
    """ncu DRAM bytes per launch, valid only for the kernel source it was taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "sparse_nvfp4_moe_b200", "csrc", "gemm_sp.cu")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return d if d.get("gemm_sp_sha256") == sha else None


def max_over_ranks(ms, world, device):
    """The slowest rank's time.  Every rank passes its own CUDA-event total; the
    replicas' whole-job time is the maximum (one all-reduce, outside the timed region)."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, steps, flops_step, max_ms):
    """Dense-equivalent TFLOP/s of the whole job: every replica does flops_step per step."""
    return world * steps * flops_step / (max_ms * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import workloads as W
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = W.CONFIGS[args.config]
    peaks = load_peaks()
    b = Bench(cfg, args.tokens, dev)
    ok = b.check_against_forward()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        step_ms, per = b.run(args.steps, max(args.warmup, 3), flush)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    clocks = clk.summary()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    S, H, I = b.S, cfg.H, cfg.I
    fl = step_flops(S, H, I)
    by = step_bytes(S, args.tokens, H, I, b.n_touched)
    flops_step = fl["gate_up"] + fl["down"]
    value = whole_job_value(world, args.steps, flops_step, total_ms)
    # roofline of the dominant kernel
    avg = {s: sum(v) / len(v) for s, v in per.items()}
    dom = max(("gemm_gate_up", "gemm_down"), key=lambda s: avg[s])
    key = "gate_up" if dom == "gemm_gate_up" else "down"
    p_fp4 = FP4_SPARSE_OVER_BF16 * peaks["bf16_tflops_sustained"]
    t_fl = fl[key] / (p_fp4 * 1e12)
    t_by = by[key] / (peaks["hbm_gbs"] * 1e9)
    dur = avg[dom] * 1e-3
    tr = traffic_record()
    traffic = None
    if tr and tr.get("workload") == f"{cfg.name}:T={args.tokens}":
        traffic = tr.get(key)
    if t_fl >= t_by:
        roof = {"bound": "tensor", "achieved": fl[key] / dur / 1e12, "peak": p_fp4, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": by[key] / dur / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof.update(kernel=f"k_grouped_gemm_sp ({key})", algorithmic_bytes=by[key], algorithmic_flops=fl[key],
                avg_launch_ms=avg[dom], peak_source=(f"{peaks['source']}: sparse FP4 = 8 x bf16 sustained "
                                                   f"{peaks['bf16_tflops_sustained']} TFLOP/s; HBM "
                                                   f"{peaks['hbm_gbs']} GB/s copy"))
    kernels = {}
    for s in b.STAGES:
        k = {"permute": "permute", "quant_act": "quant_act", "gemm_gate_up": "gate_up", "gemm_down": "down",
             "combine": "combine"}[s]
        d = avg[s] * 1e-3
        ent = {"ms": avg[s], "bytes_GBps": by[k] / d / 1e9, "hbm_frac": by[k] / d / 1e9 / peaks["hbm_gbs"]}
        if k in fl:
            ent["TFLOPs"] = fl[k] / d / 1e12
            ent["tensor_frac"] = fl[k] / d / 1e12 / p_fp4
            ent["roofline_frac"] = max(fl[k] / (p_fp4 * 1e12), by[k] / (peaks["hbm_gbs"] * 1e9)) / d
        kernels[s] = ent
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3 block scales) -> fp32 accumulate",
        "data": "synthetic (seeded bf16 N(0,0.02) weights pruned/quantised by the library; bf16 N(0,1) "
                "inputs with 1% x20 outlier channels; uniform random router logits)",
        "config": {"workload": f"{cfg.name}-shaped MoE expert layer, full path (moe_forward stages)",
                   "E": cfg.E, "k": cfg.k, "H": H, "I": I, "tokens": args.tokens, "slots": S,
                   "experts_touched": b.n_touched, "max_group": b.max_group,
                   "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "staged_equals_forward": ok,
        "clocks": clocks,
    }
    if not args.no_e2e:
        ms, h2d, d2h = b.e2e(max(3, args.steps // 4), 2)
        e2e_val = whole_job_value(world, 1, flops_step, max_over_ranks(ms, world, dev))
        out["e2e"] = {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": ms, "api": "moesq_moe_forward_host (pinned host buffers)"}
    if not args.no_sweep and world == 1:
        sweep = []
        for T in cfg.tokens:
            if T == args.tokens:
                continue
            bb = Bench(cfg, T, dev, lin=b.lin)
            st_t, per_t = bb.run(10, 3, flush)
            a = {s: sum(v) / len(v) for s, v in per_t.items()}
            f2 = step_flops(bb.S, H, I)
            y2 = step_bytes(bb.S, T, H, I, bb.n_touched)
            ms_t = sum(st_t) / len(st_t)
            row = {"tokens": T, "ms_per_step": ms_t,
                   "TFLOPs": (f2["gate_up"] + f2["down"]) / (ms_t * 1e-3) / 1e12}
            for s, k in (("gemm_gate_up", "gate_up"), ("gemm_down", "down")):
                d = a[s] * 1e-3
                row[k] = {"ms": a[s], "TFLOPs": f2[k] / d / 1e12, "GBps": y2[k] / d / 1e9,
                          "roofline_frac": max(f2[k] / (p_fp4 * 1e12), y2[k] / (peaks["hbm_gbs"] * 1e9)) / d,
                          "bound": ("tensor" if f2[k] / (p_fp4 * 1e12) > y2[k] / (peaks["hbm_gbs"] * 1e9)
                                    else "hbm")}
            sweep.append(row)
            del bb
            torch.cuda.empty_cache()
        out["sweep"] = sweep
    if not args.no_sweep and world == 1:
        d = b.dense_comparison(10, flush)
        fl_d = step_flops(b.S, H, I)
        by_w = {"gate_up": b.n_touched * 2 * I * H, "down": b.n_touched * H * I}
        out["dense_comparison"] = {
            "what": "the same gate_up (SwiGLU + requant) and down (bf16) GEMMs on the decoded dense NVFP4 "
                    "weights (dense tcgen05 MMA, 16-element scale blocks), same workload and inputs",
            **{f"{k}_ms": d[k] for k in d},
            **{f"{k}_TFLOPs": fl_d[k] / (d[k] * 1e-3) / 1e12 for k in d},
            "sparse_speedup": {k: d[k] / avg["gemm_" + k] for k in d},
            "weight_bytes_per_dense_element": {"sparse": 0.34375, "dense": 0.53125},
            "weight_bytes_touched_GB": {k: {"sparse": by_w[k] * 0.34375 / 1e9, "dense": by_w[k] * 0.53125 / 1e9}
                                        for k in by_w},
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = {k: v for k, v in cpu_baseline(cfg, args.tokens, args.cpu_slots).items()
                               if k != "seconds"}
    if int(b.status.item()) != 0:
        out["device_status"] = int(b.status.item())
    return out


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores, on a bounded per-step sample."""
    if rank != 0:
        return None
    import workloads as W
    cfg = W.CONFIGS[args.config]
    slots = 128
    vals = []
    for i in range(max(args.warmup, 0) + args.steps):
        r = cpu_baseline(cfg, args.tokens, slots)
        if i >= args.warmup:
            vals.append(r)
    tot_flops = sum(v["value"] * v["seconds"] for v in vals)
    tot_s = sum(v["seconds"] for v in vals)
    value = tot_flops / tot_s
    cb = dict(vals[-1])
    cb.pop("seconds", None)
    cb["value"] = value
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / len(vals) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64 (exact)",
            "data": "synthetic", "config": {"workload": f"{cfg.name}-shaped MoE expert layer (oracle sample)",
                                              "tokens": args.tokens, "slots_per_step": slots},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------ storage benchmark ---
# bytes per dense element moved by each storage kernel (in + out)
STORAGE_BYTES = dict(decode=0.25 + 1 / 16 + 0.5,          # packed + mask -> dense codes
                     encode=0.5 + 1 / 16 + 0.25 + 1 / 16,  # dense codes + mask hint -> packed + mask
                     repack=1 / 16 + 1 / 32 + 1 / 16 + 1 / 32)  # mask + scales -> metadata + scale blocks


def run_storage(args):
    """Every expert linear of a layer (gate_up and down of all experts) exported to
    pair-bitmask storage by the library, then per pass: decode to dense NVFP4
    codes, re-encode (checked bit-exact against the stored bytes) and repack into
    the GEMM layouts.  value = bytes moved per pass / pass time."""
    import torch

    import sparse_nvfp4_moe_b200 as M
    import workloads as W
    cfg_name = args.config if args.config != "qwen3_30b_a3b" else "kimi_k2"
    cfg = W.CONFIGS[cfg_name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    tensors = []
    split = cfg.split_gate_up_global
    for which, n_seg, kind in (("gate_up", 2 if split else 1, M.KIND_GATE_UP_SPLIT if split else M.KIND_GATE_UP),
                               ("down", 1, M.KIND_DOWN)):
        parts = []
        for e0 in range(0, cfg.E, 64):
            w = W.all_expert_weights_bf16(cfg, which, device=dev, experts=range(e0, min(cfg.E, e0 + 64)))
            parts.append(M.quantize_expert_weights(w, n_seg))
            del w
        st = {k: torch.cat([p_[k] for p_ in parts]) for k in ("packed", "mask", "scale", "g_w")}
        E, out, K = cfg.E, parts[0]["out"], parts[0]["K"]
        del parts
        torch.cuda.empty_cache()
        mb, sb = M.repack_sizes(out, K)
        u8 = dict(dtype=torch.uint8, device=dev)
        tensors.append(dict(which=which, kind=kind, E=E, out=out, K=K,
                            st=st, dense=torch.empty((E * out, K // 2), **u8),
                            packed2=torch.empty_like(st["packed"]), mask2=torch.empty_like(st["mask"]),
                            meta=torch.empty(E * mb, **u8), sf=torch.empty(E * sb, **u8),
                            alpha=torch.empty(E, dtype=torch.float32, device=dev)))
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def op(name):
        for t in tensors:
            rows = t["E"] * t["out"]
            if name == "decode":
                M.moesq_decode(t["st"]["packed"], t["st"]["mask"], t["dense"], rows, t["K"], status)
            elif name == "encode":
                M.moesq_encode(t["dense"], t["st"]["mask"], t["packed2"], t["mask2"], rows, t["K"], status)
            else:
                M.moesq_repack_meta(t["st"]["mask"], t["st"]["scale"], t["st"]["g_w"], t["E"], t["out"], t["K"],
                                    t["kind"], t["meta"], t["sf"], t["alpha"], status)

    n_elem = sum(t["E"] * t["out"] * t["K"] for t in tensors)
    for _ in range(max(args.warmup, 3)):
        for name in STORAGE_BYTES:
            op(name)
    torch.cuda.synchronize()
    exact = all(torch.equal(t["packed2"], t["st"]["packed"]) and torch.equal(t["mask2"], t["st"]["mask"])
                for t in tensors)
    per = {}
    with ClockSampler(dev.index) as clk:
        for name in STORAGE_BYTES:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for a, b in ev:
                a.record()
                op(name)
                b.record()
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
            gb = STORAGE_BYTES[name] * n_elem / 1e9
            per[name] = {"ms": ms, "GB": gb, "GBps": gb / (ms * 1e-3), "hbm_frac": gb / (ms * 1e-3) / peaks["hbm_gbs"]}
    clocks = clk.summary()
    tot_ms = sum(v["ms"] for v in per.values())
    tot_gb = sum(v["GB"] for v in per.values())
    # the inputs are resident between passes and larger than L2 (no flush needed)
    return {"metric": f"pair-bitmask storage decode + re-encode + repack GB/s, all {cfg.E} experts' "
                      f"gate_up and down ({cfg.name}-shaped, 1 B200)",
            "value": tot_gb / (tot_ms * 1e-3), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": tot_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u8 (E2M1 codes, pair bitmask, E4M3 scales)", "data": "synthetic",
            "config": {"workload": f"{cfg.name} storage: {cfg.E} experts x (gate_up [{2 * cfg.I},{cfg.H}] + "
                                   f"down [{cfg.H},{cfg.I}])", "dense_elements": n_elem,
                       "l2": "not flushed: every pass moves > 10 GB"},
            "round_trip_bit_exact": bool(exact), "per_op": per,
            "roofline": {"bound": "hbm", "achieved": tot_gb / (tot_ms * 1e-3), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": tot_gb / (tot_ms * 1e-3) / peaks["hbm_gbs"], "traffic": None},
            "device_status": int(status.item()), "clocks": clocks,
            # per step and tensor: decode 1, encode 1, repack 2 (metadata, scale blocks)
            "gpu_launches": 4 * len(tensors) * args.steps}


def main():
    args = parse_args()
    if args.storage and args.impl == "ours":
        print(json.dumps(run_storage(args)))
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res))
        return 0
    import torch.distributed as dist
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
