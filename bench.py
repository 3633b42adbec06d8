#!/usr/bin/env python
"""Benchmark of the paired-4:8 sparse NVFP4 MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config qwen3_235b_a22b] [--tokens 65536] [--no-shapes] [--no-storage]
    python bench.py --storage [--config kimi_k2]          # the storage benchmark alone
    python bench.py --traffic-csv ncu.csv --traffic-cmd "..."   # ncu DRAM bytes -> profiles/

A step is one pass of the whole routed-expert path over one synthetic batch:
permute -> NVFP4 activation quantisation -> gate_up sparse grouped GEMM with the
fused SwiGLU + NVFP4 requant epilogue -> down sparse grouped GEMM -> weighted
combine.  Weights are drawn (bf16 N(0, 0.02)), pruned, quantised and encoded to
pair-bitmask storage by the library's own kernels, then repacked.  Inputs sit
in HBM before timing; L2 is flushed (a 256 MiB write) between timed steps and
every stage is timed with CUDA events on the launch stream.

The headline line runs the largest layer shape that fits one GPU, Qwen3-235B-A22B
at 65536 tokens, as the full path.  Its `shapes` key holds the GEMM and step rows
of every layer shape and token count (Qwen3-30B-A3B, Qwen3.5-397B-A17B,
Qwen3-235B-A22B, Kimi-K2), with each GEMM also timed back to back over rotated
weight and activation copies (so that every launch streams its operands from HBM,
not L2); its `storage` key holds the Kimi-K2 storage benchmark.

Metric: dense-equivalent TFLOP/s (2*S*2I*H + 2*S*H*I per step, S = tokens*k),
whole job over all ranks.  Multi-GPU runs (one process per GPU under torchrun) are
expert parallel by default (weak scaling): rank r holds a contiguous 1/N of the
experts and routes its own batch of --tokens tokens, and every step sends each
routed slot's NVFP4 codes and scales to its expert's rank and the bf16 outputs back
(NCCL all-to-all).  --replicas runs N independent copies of the one-GPU path instead.

--impl reference times the CPU oracle (numpy, exact integer products through
float64) on a bounded sample of the same workload on the host cores; it is a
deliberately slow program.
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
def kernels_per_step(cfg, T):
    """Library kernels one step launches: the permute (1 kernel up to 1024 slots, else 3),
    the routed quant (a second, in-place kernel rearranges its row-major scales into the
    tensor-core blocks when K % 1024 == 0, k <= 32 and the codes written reach 64 MiB),
    the two GEMMs and the combine."""
    perm = 1 if T * cfg.k <= 1024 else 3
    quant = 2 if cfg.H % 1024 == 0 and cfg.k <= 32 and T * cfg.k * (cfg.H // 2) >= (64 << 20) else 1
    return perm + quant + 3
L2_BYTES = 126 * 1024 * 1024    # B200 L2
DEFAULT_CONFIG, DEFAULT_TOKENS = "qwen3_235b_a22b", 65536
SHAPE_CONFIGS = ("qwen3_30b_a3b", "qwen3_5_397b_a17b", "qwen3_235b_a22b", "kimi_k2")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=None, help=f"layer shape (default {DEFAULT_CONFIG})")
    ap.add_argument("--tokens", type=int, default=DEFAULT_TOKENS)
    ap.add_argument("--no-shapes", action="store_true", help="skip the rows of every layer shape and token count")
    ap.add_argument("--shape-configs", default=",".join(SHAPE_CONFIGS))
    ap.add_argument("--no-storage", action="store_true", help="skip the Kimi-K2 storage benchmark key")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense comparison GEMMs")
    ap.add_argument("--no-fused", action="store_true", help="skip the fused down + combine comparison")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-slots", type=int, default=256, help="slots in the CPU-baseline sample")
    ap.add_argument("--storage", action="store_true",
                    help="storage benchmark instead: decode / re-encode / repack every expert's "
                         "pair-bitmask tensors of --config (default kimi_k2 with this flag)")
    ap.add_argument("--traffic-csv", default=None,
                    help="write profiles/traffic.json from this ncu CSV (dram__bytes_read.sum and "
                         "dram__bytes_write.sum of the GEMM launches) and exit")
    ap.add_argument("--traffic-cmd", default="", help="the command the ncu CSV came from (recorded)")
    ap.add_argument("--ep", action="store_true",
                    help="expert-parallel mode even on one rank (under torchrun), the default for N > 1")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1 GPUs: N independent replicas of the one-GPU path instead of expert parallelism")
    a = ap.parse_args()
    if a.config is None:
        a.config = "kimi_k2" if a.storage else DEFAULT_CONFIG
    return a


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def fp4_peaks(peaks):
    """Dense-equivalent sparse FP4 tensor peaks, burst and sustained: the larger of 8 x
    the measured bf16 GEMM rate (the nominal sparse-FP4 / bf16 ratio, 18 / 2.25 PFLOP/s)
    and the sparse-MMA rate measured on this GPU (`fp4sp_micro`, a burst figure; its
    sustained counterpart is scaled by the bf16 sustained / burst ratio)."""
    b8 = FP4_SPARSE_OVER_BF16 * peaks["bf16_tflops"]
    s8 = FP4_SPARSE_OVER_BF16 * peaks["bf16_tflops_sustained"]
    micro = peaks.get("fp4sp_micro") or 0.0
    return max(b8, micro), max(s8, micro * peaks["bf16_tflops_sustained"] / peaks["bf16_tflops"])


def measure_fp4_peak(peaks):
    """The sparse-MMA microbenchmark (moesq_measure_sparse_mma_peak: every CTA pair issues
    back-to-back N = 256 sparse FP4 MMAs on operands resident in shared memory and TMEM)
    recorded into `peaks`; the GEMM rooflines use the larger of it and 8 x bf16."""
    import sparse_nvfp4_moe_b200 as M
    peaks["fp4sp_micro"] = max(M.moesq_measure_sparse_mma_peak(4000, 256) for _ in range(3))
    return peaks


def classify(flops, nbytes, weight_bytes, peaks):
    """Roofline of one GEMM launch: (bound, roofline time s, class, target).  A row is
    decode-sized when HBM binds it and weights are at least half its bytes (target: 70%
    of HBM), else prefill-sized (target: 60% of its roofline)."""
    p_burst, _ = fp4_peaks(peaks)
    t_fl = flops / (p_burst * 1e12)
    t_by = nbytes / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if t_fl > t_by else "hbm"
    decode = bound == "hbm" and weight_bytes >= 0.5 * nbytes
    return bound, max(t_fl, t_by), ("decode-sized" if decode else "prefill-sized"), (0.70 if decode else 0.60)


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

    def rotated_gemm_ms(self, which, launches=40, replays=3):
        """Per-launch time of one grouped GEMM launched back to back inside a CUDA graph,
        cycling through R rotation slots so that consecutive launches read operands L2
        does not hold.  Slot i runs on weight copy i % C and on the routing relabelled by
        a seeded permutation of the experts (the same group sizes on other experts), with
        its own activations; R * (weight bytes one launch touches) and C * (all the
        layer's weight bytes) both reach 3 x L2.  Returns (ms per launch, R, C)."""
        torch, M, cfg = self.torch, self.M, self.cfg
        lin = self.lin[which]
        per_elem = lin.out * lin.K * B_W
        touched, whole = self.n_touched * per_elem, cfg.E * per_elem
        C = int(min(8, max(1, -(-3 * L2_BYTES // int(whole)))))
        R = int(min(64, max(C, -(-3 * L2_BYTES // max(1, int(touched))))))
        lins = [lin] + [M.ExpertLinear(lin.packed.clone(), lin.meta.clone(), lin.sf.clone(), lin.alpha_w.clone(),
                                       lin.E, lin.out, lin.K, lin.kind) for _ in range(C - 1)]
        slots = []
        gen = torch.Generator(device="cpu")
        for i in range(R):
            if i == 0:
                sl = dict(eo=self.eo, po=self.po, a_codes=self.a_codes, a_sf=self.a_sf, h_codes=self.h_codes,
                          h_sf=self.h_sf)
            else:
                gen.manual_seed(1000 + i)
                perm = torch.randperm(cfg.E, generator=gen).to(self.dev)
                ids = perm[self.ids.long()].to(torch.int32).contiguous()
                i32 = dict(dtype=torch.int32, device=self.dev)
                sl = dict(eo=torch.empty(cfg.E + 1, **i32), po=torch.empty(cfg.E + 1, **i32),
                          a_codes=torch.empty_like(self.a_codes), a_sf=torch.empty_like(self.a_sf),
                          h_codes=torch.empty_like(self.h_codes), h_sf=torch.empty_like(self.h_sf))
                st, ts = torch.empty_like(self.slot_token), torch.empty_like(self.token_slot)
                M.moesq_permute(ids, self.T, cfg.k, cfg.E, sl["eo"], sl["po"], st, ts, self.perm_ws, self.perm_ws_n,
                                self.status)
                M.moesq_quant_act_routed(self.x.view(torch.uint16), self.T, cfg.H, ids, ts, cfg.k, sl["eo"], sl["po"],
                                         cfg.E, self.g_in_gu, sl["a_codes"], sl["a_sf"])
                if which == "down":
                    M.moesq_grouped_gemm(self.lin["gate_up"].struct, sl["a_codes"], sl["a_sf"], self.g_in_gu,
                                         sl["eo"], sl["po"], self.S, self.P, M.EPI_SWIGLU_NVFP4, self.g_in_dn,
                                         sl["h_codes"], sl["h_sf"], d_status=self.status)
                    del sl["a_codes"], sl["a_sf"]
            slots.append(sl)
        out_h = (torch.empty_like(self.h_codes), torch.empty_like(self.h_sf))
        out_y = torch.empty_like(self.y)

        def launch(i):
            sl, ln = slots[i], lins[i % C]
            if which == "gate_up":
                M.moesq_grouped_gemm(ln.struct, sl["a_codes"], sl["a_sf"], self.g_in_gu, sl["eo"], sl["po"], self.S,
                                     self.P, M.EPI_SWIGLU_NVFP4, self.g_in_dn, out_h[0], out_h[1],
                                     d_status=self.status)
            else:
                M.moesq_grouped_gemm(ln.struct, sl["h_codes"], sl["h_sf"], self.g_in_dn, sl["eo"], sl["po"], self.S,
                                     self.P, M.EPI_BF16, None, out_y.view(torch.uint16), None, d_status=self.status)

        reps = max(1, -(-launches // R))
        for i in range(R):
            launch(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                for i in range(R):
                    launch(i)
        stream = torch.cuda.current_stream()
        g.replay()
        torch.cuda.synchronize()
        ms = []
        for _ in range(replays):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b) / (reps * R))
        del g, slots, lins
        torch.cuda.empty_cache()
        return statistics.median(ms), R, C

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

    def fused_combine(self, steps, flush):
        """The down GEMM with the weighted combine fused into its epilogue
        (moesq_grouped_gemm_down_combine) against the down GEMM plus the separate
        combine, each as one graph after an L2 flush; and whether the fused output is
        bit-identical to the staged one."""
        torch, M = self.torch, self.M
        cfg, T = self.cfg, self.T
        for s_ in self.STAGES:
            getattr(self, s_)()
        y = torch.empty_like(self.y)
        out = torch.empty_like(self.out)
        arrivals = torch.empty(T * (cfg.H // 128), dtype=torch.int32, device=self.dev)

        def fused():
            M.moesq_grouped_gemm_down_combine(self.lin["down"].struct, self.h_codes, self.h_sf, self.g_in_dn, self.eo,
                                              self.po, self.S, self.P, self.slot_token, self.token_slot, self.w,
                                              T, cfg.k, y.view(torch.uint16), out.view(torch.uint16), arrivals,
                                              self.status)

        def staged():
            self.gemm_down()
            self.combine()

        fused()
        torch.cuda.synchronize()
        same = bool(torch.equal(out.view(torch.int16), self.out.view(torch.int16)))
        graphs = {}
        for name, fn in (("down_plus_combine", staged), ("fused", fused)):
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
        return res, same

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


def host_cpu():
    """Host cores this process may use and the CPU model (from /proc/cpuinfo)."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return {"nproc": n, "model": model}


class OracleSample:
    """A bounded sample of the workload for timing the oracle: the most-loaded expert's
    routed slots (up to n) of the layer at T tokens, with that expert's weights exported
    to pair-bitmask storage by the oracle (preparation, not timed)."""

    def __init__(self, cfg, T, n_slots):
        import numpy as np

        import workloads as W
        from oracle import routing as R
        from oracle import storage as S
        ids, _ = W.routing(cfg, T)
        perm = R.permute(np.asarray(ids), cfg.E)
        counts = np.diff(perm["expert_offsets"])
        self.e = e = int(np.argmax(counts))
        self.count = int(counts[e])
        self.n = n = int(min(n_slots, counts[e]))
        rows = perm["slot_token"][perm["expert_offsets"][e]:perm["expert_offsets"][e] + n]
        self.x = W.layer_input_bf16(cfg, T).float().numpy()[rows]
        self.n_seg = 2 if cfg.split_gate_up_global else 1
        self.gu = S.quantize_weight(W.expert_weights_bf16(cfg, e, "gate_up").float().numpy(), self.n_seg)
        self.dn = S.quantize_weight(W.expert_weights_bf16(cfg, e, "down").float().numpy(), 1)
        self.cfg, self.T = cfg, T
        self.flops = 2.0 * n * (2 * cfg.I * cfg.H + cfg.H * cfg.I)

    def run(self, threads=None):
        """quantise -> exact gate_up -> SwiGLU -> requant -> exact down for the sample's
        slots.  threads: BLAS threads of numpy's float64 products (None: all host cores).
        Returns (seconds, threads used)."""
        import numpy as np
        from threadpoolctl import threadpool_info, threadpool_limits

        from oracle import gemm as G
        from oracle import nvfp4 as N
        from oracle import storage as S
        cfg, gu, dn, n = self.cfg, self.gu, self.dn, self.n
        with threadpool_limits(limits=threads):
            blas = [i for i in threadpool_info() if i.get("user_api") == "blas"]
            used = max((int(i.get("num_threads", 1)) for i in blas), default=1)
            t0 = time.perf_counter()
            g_in = np.float32(np.abs(self.x).max() / 2688.0)
            ac, asf = N.quantize_groups(self.x, g_in)
            sc = gu["scale"].copy()
            if self.n_seg == 2:
                sc[cfg.I:] = S.fold_up_scales(sc[cfg.I:], gu["g"][0], gu["g"][1])
            Wg = G.dequant_int(N.unpack_codes(S.decode(gu["packed"], gu["mask"])), sc)
            acc, _ = G.grouped_gemm_exact([Wg], [gu["g"][0]], G.dequant_int(ac, asf), np.float32([g_in]),
                                          np.array([0, n]))
            h = G.swiglu(acc)
            g_dn = np.float32(np.abs(h).max() / 2688.0)
            hc, hs = N.quantize_groups(h.astype(np.float32), g_dn)
            G.grouped_gemm_exact([G.weight_int(dn)], [dn["g"][0]], G.dequant_int(hc, hs), np.float32([g_dn]),
                                 np.array([0, n]))
            return time.perf_counter() - t0, used

    def describe(self, dt, used):
        return (f"expert {self.e} ({self.count} routed slots) of the {self.cfg.name}-shaped layer at T={self.T}: "
                f"quantise, exact gate_up (integer products through float64), SwiGLU, requant, exact down for "
                f"{self.n} slots ({self.flops / 1e9:.1f} dense-equiv GFLOP in {dt:.2f} s on {used} BLAS "
                f"thread(s); weight export not timed)")


def cpu_baseline(cfg, T, n_slots, threads=None):
    """The oracle as it stands, timed once on a bounded sample (OracleSample)."""
    smp = OracleSample(cfg, T, n_slots)
    smp.run(threads)                 # first call pages in the BLAS
    dt, used = smp.run(threads)
    hc = host_cpu()
    return dict(value=smp.flops / dt / 1e12, unit=UNIT, cores=used, kind="oracle", sample=smp.describe(dt, used),
                nproc=hc["nproc"], cpu_model=hc["model"], seconds=dt)


def traffic_record():
    """ncu DRAM bytes per launch, valid only for the kernel source it was taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    return d if d.get("gemm_sp_sha256") == gemm_source_sha() else None


def gemm_source_sha():
    src = os.path.join(ROOT, "sparse_nvfp4_moe_b200", "csrc", "gemm_sp.cu")
    return hashlib.sha256(open(src, "rb").read()).hexdigest()


def write_traffic(csv_path, command, workload):
    """profiles/traffic.json from an ncu CSV of the grouped-GEMM launches (metrics
    dram__bytes_read.sum and dram__bytes_write.sum, one row per launch and metric):
    mean DRAM bytes per launch of the gate_up (SwiGLU epilogue) and down (bf16) GEMMs,
    stamped with the hash of the kernel source they were taken on."""
    import collections
    import csv
    rows = list(csv.reader(open(csv_path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr, data = rows[hi], rows[hi + 1:]
    ki, mi, vi, ui, idi = (hdr.index(c) for c in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit", "ID"))
    unit = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    per = collections.defaultdict(dict)
    for r in data:
        if len(r) <= vi or not r[vi]:
            continue
        per[(r[idi], r[ki])][r[mi]] = float(r[vi].replace(",", "")) * unit.get(r[ui], 1)
    res = {}
    for (_, name), m in per.items():
        key = "gate_up" if "k_grouped_gemm_sp<2," in name else ("down" if "k_grouped_gemm_sp<1," in name else None)
        if key is None or "dram__bytes_read.sum" not in m:
            continue
        res.setdefault(key, []).append(m["dram__bytes_read.sum"] + m.get("dram__bytes_write.sum", 0.0))
    out = {"workload": workload, "gemm_sp_sha256": gemm_source_sha(), "command": command,
           "launches": {k: len(v) for k, v in res.items()}}
    for k, v in res.items():
        out[k] = sum(v) / len(v)
    path = os.path.join(ROOT, "profiles", "traffic.json")
    json.dump(out, open(path, "w"), indent=1)
    return out


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


def gemm_row(b, key, ms, isolated_ms, peaks, rot=None):
    """One GEMM's figures on one layer shape and token count."""
    cfg = b.cfg
    fl = step_flops(b.S, cfg.H, cfg.I)[key]
    by = step_bytes(b.S, b.T, cfg.H, cfg.I, b.n_touched)[key]
    wb = b.n_touched * (2 * cfg.I * cfg.H if key == "gate_up" else cfg.H * cfg.I) * B_W
    bound, t_roof, cls, target = classify(fl, by, wb, peaks)
    p_burst, p_sust = fp4_peaks(peaks)
    d = ms * 1e-3
    row = {"ms": ms, "isolated_ms": isolated_ms, "TFLOPs": fl / d / 1e12, "GBps": by / d / 1e9,
           "hbm_frac": by / d / 1e9 / peaks["hbm_gbs"], "tensor_frac": fl / d / 1e12 / p_burst,
           "roofline_frac": t_roof / d, "bound": bound, "class": cls, "target": target,
           "meets_target": (by / d / 1e9 / peaks["hbm_gbs"] if cls == "decode-sized" else t_roof / d) >= target,
           "algorithmic_bytes": by, "weight_bytes": wb, "flops": fl}
    if rot is not None:
        row["rotation"] = {"slots": rot[0], "weight_copies": rot[1]}
    return row


def shape_rows(b_main, cfg_names, flush, peaks, dev):
    """GEMM and step rows of every layer shape and token count (one GPU)."""
    import torch

    import workloads as W
    rows = []
    for name in cfg_names:
        cfg = W.CONFIGS[name]
        lin = b_main.lin if cfg.name == b_main.cfg.name else None
        for T in cfg.tokens:
            if cfg.name == b_main.cfg.name and T == b_main.T:
                bb = b_main
            else:
                bb = Bench(cfg, T, dev, lin=lin)
                lin = bb.lin
            st_t, per_t = bb.run(5, 3, flush)
            iso = {s: statistics.median(v) for s, v in per_t.items()}
            ms_t = statistics.median(st_t)
            f2 = step_flops(bb.S, cfg.H, cfg.I)
            row = {"config": cfg.name, "tokens": T, "slots": bb.S, "experts_touched": bb.n_touched,
                   "max_group": bb.max_group, "ms_per_step": ms_t,
                   "TFLOPs": (f2["gate_up"] + f2["down"]) / (ms_t * 1e-3) / 1e12,
                   "tokens_per_s": T / (ms_t * 1e-3)}
            for st, key in (("gemm_gate_up", "gate_up"), ("gemm_down", "down")):
                ms_r, R, C = bb.rotated_gemm_ms(key)
                row[key] = gemm_row(bb, key, ms_r, iso[st], peaks, (R, C))
            rows.append(row)
            if bb is not b_main:
                del bb
            torch.cuda.empty_cache()
        del lin
        torch.cuda.empty_cache()
    return rows


def run_ours(args, rank, world, local_rank):
    import torch

    import workloads as W
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = W.CONFIGS[args.config]
    peaks = measure_fp4_peak(load_peaks())
    p_burst, p_sust = fp4_peaks(peaks)
    b = Bench(cfg, args.tokens, dev)
    ok = b.check_against_forward()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        step_ms, per = b.run(args.steps, max(args.warmup, 3), flush)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    clocks = clk.summary()
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    S, H, I = b.S, cfg.H, cfg.I
    fl = step_flops(S, H, I)
    by = step_bytes(S, args.tokens, H, I, b.n_touched)
    flops_step = fl["gate_up"] + fl["down"]
    value = whole_job_value(world, args.steps, flops_step, total_ms)
    # roofline of the dominant kernel, timed alone in its own graph after an L2 flush
    avg = {s: sum(v) / len(v) for s, v in per.items()}
    dom = max(("gemm_gate_up", "gemm_down"), key=lambda s: avg[s])
    key = "gate_up" if dom == "gemm_gate_up" else "down"
    wb = b.n_touched * (2 * I * H if key == "gate_up" else H * I) * B_W
    bound, _, cls, target = classify(fl[key], by[key], wb, peaks)
    dur = avg[dom] * 1e-3
    tr = traffic_record()
    traffic = None
    if tr and tr.get("workload") == f"{cfg.name}:T={args.tokens}":
        traffic = tr.get(key)
    if bound == "tensor":
        roof = {"bound": "tensor", "achieved": fl[key] / dur / 1e12, "peak": p_burst, "unit": "TFLOP/s"}
        roof["frac_of_sustained_peak"] = roof["achieved"] / p_sust
    else:
        roof = {"bound": "hbm", "achieved": by[key] / dur / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof.update(kernel=f"k_grouped_gemm_sp ({key})", algorithmic_bytes=by[key], algorithmic_flops=fl[key],
                avg_launch_ms=avg[dom], row_class=cls, target=target,
                peak_source=(f"sparse FP4 (dense-equivalent) = max(sparse-MMA microbenchmark measured in this "
                             f"run {peaks['fp4sp_micro']:.0f} TFLOP/s, 8 x {peaks['source']} bf16 GEMM burst "
                             f"{peaks['bf16_tflops']} = {FP4_SPARSE_OVER_BF16 * peaks['bf16_tflops']:.0f}) = "
                             f"{p_burst:.0f} TFLOP/s (sustained {p_sust:.0f}); HBM {peaks['hbm_gbs']} GB/s copy "
                             f"({peaks['source']})"),
                sparse_mma_microbenchmark_tflops=peaks["fp4sp_micro"])
    kernels = {}
    for s_ in b.STAGES:
        k = {"permute": "permute", "quant_act": "quant_act", "gemm_gate_up": "gate_up", "gemm_down": "down",
             "combine": "combine"}[s_]
        d = avg[s_] * 1e-3
        ent = {"ms": avg[s_], "bytes_GBps": by[k] / d / 1e9, "hbm_frac": by[k] / d / 1e9 / peaks["hbm_gbs"]}
        if k in fl:
            ent["TFLOPs"] = fl[k] / d / 1e12
            ent["tensor_frac"] = fl[k] / d / 1e12 / p_burst
            ent["roofline_frac"] = max(fl[k] / (p_burst * 1e12), by[k] / (peaks["hbm_gbs"] * 1e9)) / d
        kernels[s_] = ent
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3 block scales) -> fp32 accumulate",
        "data": ("synthetic (seeded bf16 N(0,0.02) weights pruned/quantised by the library; bf16 N(0,1) inputs"
                 + ("; 1% x20 outlier channels" if cfg.outlier_channels else "")
                 + f"; {cfg.routing} router logits)"),
        "config": {"workload": (f"{cfg.name}-shaped MoE expert layer ({cfg.E} experts, top-{cfg.k}, hidden {H}, "
                                f"intermediate {I}) at {args.tokens} tokens, the full moe_forward path: permute, "
                                f"activation quant, gate_up + SwiGLU + NVFP4 requant, down, weighted combine"),
                   "E": cfg.E, "k": cfg.k, "H": H, "I": I, "tokens": args.tokens, "slots": S,
                   "experts_touched": b.n_touched, "max_group": b.max_group,
                   "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": kernels_per_step(cfg, args.tokens) * args.steps,
        "staged_equals_forward": ok,
        "clocks": clocks,
    }
    if not args.no_e2e:
        ms, h2d, d2h = b.e2e(max(3, args.steps // 4), 2)
        e2e_val = whole_job_value(world, 1, flops_step, max_over_ranks(ms, world, dev))
        out["e2e"] = {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": ms, "api": "moesq_moe_forward_host (pinned host buffers)"}
    if world == 1 and not args.no_dense:
        d = b.dense_comparison(10, flush)
        by_w = {"gate_up": b.n_touched * 2 * I * H, "down": b.n_touched * H * I}
        out["dense_comparison"] = {
            "what": "the same gate_up (SwiGLU + requant) and down (bf16) GEMMs on the decoded dense NVFP4 "
                    "weights (dense tcgen05 MMA, 16-element scale blocks), same workload and inputs",
            **{f"{k}_ms": d[k] for k in d},
            **{f"{k}_TFLOPs": fl[k] / (d[k] * 1e-3) / 1e12 for k in d},
            "sparse_speedup": {k: d[k] / avg["gemm_" + k] for k in d},
            "weight_bytes_per_dense_element": {"sparse": 0.34375, "dense": 0.53125},
            "weight_bytes_touched_GB": {k: {"sparse": by_w[k] * 0.34375 / 1e9, "dense": by_w[k] * 0.53125 / 1e9}
                                        for k in by_w},
        }
    if world == 1 and not args.no_fused:
        d, same = b.fused_combine(10, flush)
        out["fused_combine"] = {
            "what": "down GEMM with the weighted combine fused into its epilogue (per-token arrival counts, the "
                    "completing arrival sums the k rows in j order) vs the down GEMM and the separate combine",
            "down_plus_combine_ms": d["down_plus_combine"], "fused_ms": d["fused"],
            "fused_speedup": d["down_plus_combine"] / d["fused"], "bit_identical": same,
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        one = cpu_baseline(cfg, args.tokens, args.cpu_slots, threads=1)
        allc = cpu_baseline(cfg, args.tokens, 8 * args.cpu_slots, threads=None)
        cb = {k: v for k, v in allc.items() if k != "seconds"}
        cb["single_thread"] = {k: v for k, v in one.items() if k not in ("seconds", "kind", "nproc", "cpu_model")}
        out["cpu_baseline"] = cb
    if world == 1 and not args.no_shapes:
        names = [n for n in args.shape_configs.split(",") if n]
        out["shapes"] = shape_rows(b, names, flush, peaks, dev)
        out["shapes_method"] = (
            "per row: ms_per_step = the whole path as one CUDA graph after an L2 flush (median of 5); per GEMM: "
            "ms = one launch of a CUDA graph of >= 40 back-to-back launches that cycle through rotation slots "
            "(relabelled routings and weight copies, >= 3 x L2 of distinct operands); isolated_ms = the GEMM "
            "alone in its own graph after an L2 flush (includes graph launch and cold start); fractions against "
            "the measured HBM copy and 8 x the measured bf16 burst peak; decode-sized rows (HBM-bound, weights "
            ">= half the bytes) target 70% of HBM, the others 60% of their roofline")
    if int(b.status.item()) != 0:
        out["device_status"] = int(b.status.item())
    del b
    torch.cuda.empty_cache()
    if world == 1 and not args.no_storage:
        a2 = argparse.Namespace(**vars(args))
        a2.config, a2.steps, a2.warmup = "kimi_k2", 5, 3
        st = run_storage(a2)
        out["storage"] = {k: st[k] for k in ("metric", "value", "unit", "ms_per_step", "round_trip_bit_exact",
                                             "per_op", "config", "device_status")}
        out["storage"]["hbm_frac"] = st["roofline"]["frac"]
    return out


def ep_launches(T, k, n_recv):
    """Library kernels one expert-parallel step launches on a rank: permute of its
    tokens (1 kernel up to 1024 slots, else 3), quantisation, permute of the received
    slots (same rule), gather into the operand layout, the two GEMMs, the gather back
    to the received order and the weighted combine."""
    perm = lambda n: 1 if n <= 1024 else 3
    return perm(T * k) + 1 + (perm(n_recv) + 1 + 2 + 1 if n_recv > 0 else 0) + 1


def run_ep(args, rank, world, local_rank):
    """Expert parallelism over the ranks (one process per GPU, NCCL): rank r holds the
    contiguous expert range [E r / N, E (r+1) / N) and routes its own batch of T tokens;
    each step dispatches every routed slot's NVFP4 codes and scales to its expert's rank
    and brings the bf16 down outputs back for the j-order combine
    (sparse_nvfp4_moe_b200.ep.ExpertParallelMoE).  Weak scaling: T tokens per rank."""
    import dataclasses

    import torch
    import torch.distributed as dist

    import sparse_nvfp4_moe_b200 as M
    import workloads as W
    from sparse_nvfp4_moe_b200.ep import DeviceCompute, ExpertParallelMoE, expert_ranges
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = W.CONFIGS[args.config]
    T, H, I, E, k = args.tokens, cfg.H, cfg.I, cfg.E, cfg.k
    lo, hi = expert_ranges(E, world)[rank]
    n_seg = 2 if cfg.split_gate_up_global else 1
    lin = {}
    for which, ns, kd in (("gate_up", n_seg, M.KIND_GATE_UP_SPLIT if n_seg == 2 else M.KIND_GATE_UP),
                          ("down", 1, M.KIND_DOWN)):
        w = W.all_expert_weights_bf16(cfg, which, device=dev, experts=range(lo, hi))
        st = M.quantize_expert_weights(w, ns)
        del w
        lin[which] = M.ExpertLinear.from_storage(st, kd)
        del st
    # this rank's tokens: the layer's generator reseeded per rank (the weights keep the layer's seed)
    tcfg = dataclasses.replace(cfg, seed=cfg.seed + 7919 * (rank + 1))
    x = W.layer_input_bf16(tcfg, T, device=dev)
    ids, tw = W.routing(tcfg, T, device=dev)
    ids, tw = ids.contiguous(), tw.contiguous()
    # one static input global for every rank (the largest amax/(6*448) over the ranks'
    # batches) and fixed down-input globals: the values do not change the work
    g = torch.tensor([W.activation_global_scale_input(x)], dtype=torch.float32, device=dev)
    dist.all_reduce(g, op=dist.ReduceOp.MAX)
    g_all = g.expand(E).contiguous()
    g_dn = torch.full((hi - lo,), 0.01, dtype=torch.float32, device=dev)
    local = M.MoELayer(k, lin["gate_up"], lin["down"], g_all[lo:hi].contiguous(), g_dn)
    moe = ExpertParallelMoE(E, k, H, DeviceCompute(local, g_all))
    # slots this rank sends to every rank (its routing is fixed over the steps)
    owner = torch.bucketize(ids.long().flatten(), torch.tensor([h for _, h in expert_ranges(E, world)], device=dev),
                            right=True)
    send = torch.bincount(owner, minlength=world).to(torch.int64)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send)
    send_h, recv_h = send.cpu().tolist(), recv.cpu().tolist()
    remote_out = sum(send_h) - send_h[rank]
    remote_in = sum(recv_h) - recv_h[rank]
    for _ in range(max(args.warmup, 3)):
        moe.forward(x, ids, tw)
    torch.cuda.synchronize()
    dist.barrier()
    stream = torch.cuda.current_stream()
    with ClockSampler(local_rank) as clk:
        dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            moe.forward(x, ids, tw)
        b.record(stream)
        b.synchronize()
        dist.barrier()
    clocks = clk.summary()
    total_ms = max_over_ranks(a.elapsed_time(b), world, dev)
    fl = step_flops(T * k, H, I)
    flops_step = fl["gate_up"] + fl["down"]
    value = whole_job_value(world, args.steps, flops_step, total_ms)
    # end to end: the batch and its routing from pinned host memory, the output back
    hx, hids, hw = x.cpu().pin_memory(), ids.cpu().pin_memory(), tw.cpu().pin_memory()
    hout = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    n_e2e = max(3, args.steps // 4)
    for _ in range(2):
        hout.copy_(moe.forward(hx.to(dev, non_blocking=True), hids.to(dev, non_blocking=True),
                               hw.to(dev, non_blocking=True)), non_blocking=True)
    torch.cuda.synchronize()
    dist.barrier()
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a2.record(stream)
    for _ in range(n_e2e):
        hout.copy_(moe.forward(hx.to(dev, non_blocking=True), hids.to(dev, non_blocking=True),
                               hw.to(dev, non_blocking=True)), non_blocking=True)
    b2.record(stream)
    b2.synchronize()
    e2e_ms = max_over_ranks(a2.elapsed_time(b2) / n_e2e, world, dev)
    per_slot_dispatch = H // 2 + H // 32 + 4      # codes, scales, local expert id
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3 block scales) -> fp32 accumulate",
        "data": "synthetic (seeded per rank; bf16 N(0,0.02) weights pruned/quantised by the library)",
        "config": {"workload": (f"{cfg.name}-shaped MoE expert layer ({E} experts, top-{k}, hidden {H}, "
                                f"intermediate {I}), expert parallel over {world} GPUs: {T} tokens per rank, "
                                f"experts [{lo}, {hi}) on rank {rank} of a contiguous split"),
                   "E": E, "k": k, "H": H, "I": I, "tokens_per_rank": T, "slots_per_rank": T * k,
                   "l2": "not flushed: every step's operands exceed L2", "parallelism": f"ep{world}"},
        "ep": {"dispatch_bytes_rank0": remote_out * per_slot_dispatch, "combine_bytes_rank0": remote_in * H * 2,
               "slots_sent_rank0": send_h, "slots_received_rank0": recv_h,
               "exchange": "torch.distributed.all_to_all_single (NCCL) of NVFP4 codes+scales out, bf16 rows back"},
        "e2e": {"value": whole_job_value(world, 1, flops_step, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": hx.numel() * 2 + hids.numel() * 4 + hw.numel() * 4,
                "d2h_bytes_per_step": hout.numel() * 2, "ms_per_step": e2e_ms,
                "api": "ExpertParallelMoE.forward on host-copied inputs (pinned)"},
        "gpu_launches": args.steps * ep_launches(T, k, sum(recv_h)),
        "clocks": clocks,
    }
    if int(moe.compute.status.item()) != 0:
        out["device_status"] = int(moe.compute.status.item())
    return out


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores, on a bounded per-step sample."""
    if rank != 0:
        return None
    import workloads as W
    cfg = W.CONFIGS[args.config]
    slots = 128
    smp = OracleSample(cfg, args.tokens, slots)
    for _ in range(max(args.warmup, 0)):
        smp.run()
    times = []
    used = 1
    for _ in range(args.steps):
        dt, used = smp.run()
        times.append(dt)
    tot_s = sum(times)
    value = smp.flops * len(times) / tot_s / 1e12
    hc = host_cpu()
    cb = {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
          "sample": smp.describe(tot_s / len(times), used) + " per step", "nproc": hc["nproc"],
          "cpu_model": hc["model"]}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / len(times) * 1e3,
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
    cfg = W.CONFIGS[args.config]
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
    if args.traffic_csv:
        print(json.dumps(write_traffic(args.traffic_csv, args.traffic_cmd, f"{args.config}:T={args.tokens}")))
        return 0
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
    if world > 1 or (args.ep and "RANK" in os.environ):
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        use_ep = (world > 1 and not args.replicas) or (args.ep and dist.is_initialized())
        res = run_ep(args, rank, world, local_rank) if use_ep else run_ours(args, rank, world, local_rank)
    finally:
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
