"""Seeded synthetic inputs for the sparse NVFP4 MoE expert layer.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no pruning, no quantisation, no storage encoding, no
GEMM). Both the CPU oracle and the CUDA path take their inputs from here.

Workload shapes follow the expert shapes of the model families named in the
MoESQ repository README ("Supported models" table) and on the model cards
(Qwen3-30B-A3B, Qwen3.5-397B-A17B, Kimi K2).  The pages publish no data; every
tensor below is synthetic:

* expert weights: bf16 draws of N(0, 0.02), fused gate_up ``[2I, H]`` (gate
  rows first) and down ``[H, I]`` per expert;
* layer input ``x``: bf16 N(0, 1); the Qwen3-30B-A3B-shaped layer scales a
  seeded 1 % of the hidden channels by 20 before the bf16 rounding;
* router: fp32 logits N(0, 1), plus for the Zipf-routed layers a per-expert
  bias ``ln p_e`` with ``p_e`` proportional to ``rank_e ** -1.1`` over a
  seeded permutation of the experts; softmax, top-k (ties to the lower expert
  id), weights renormalised over the chosen k.  The router is not part of the
  compressed path (the model cards keep ``mlp.gate`` in BF16), so its output
  (``topk_ids``, ``topk_w``) is an input here.

Every draw is keyed by ``(seed, tensor id, expert)`` so any single expert can
be regenerated on its own, on the CPU or on a CUDA device.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

# tensor ids used in the draw keys
_T_GATE_UP, _T_DOWN, _T_X, _T_LOGITS, _T_BIAS, _T_OUTLIER = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    seed: int
    E: int            # routed experts
    k: int            # experts per token
    H: int            # hidden size (K of gate_up, out of down)
    I: int            # expert intermediate size
    tokens: tuple     # token counts of the sweep
    routing: str      # "uniform" or "zipf"
    split_gate_up_global: bool   # separate global scales for gate and up
    outlier_channels: float = 0.0  # fraction of hidden channels scaled x20


CONFIGS = {
    "tiny": LayerConfig("tiny", 1, 8, 2, 256, 128, (64,), "uniform", False),
    "qwen3_30b_a3b": LayerConfig("qwen3_30b_a3b", 2, 128, 8, 2048, 768,
                                 (1, 8, 64, 512, 4096, 16384), "uniform", True,
                                 outlier_channels=0.01),
    "qwen3_5_397b_a17b": LayerConfig("qwen3_5_397b_a17b", 3, 512, 10, 4096, 1024,
                                     (1, 16, 256, 4096, 32768), "zipf", True),
    "qwen3_235b_a22b": LayerConfig("qwen3_235b_a22b", 4, 128, 8, 4096, 1536,
                                   (8192, 65536), "uniform", True),
    "kimi_k2": LayerConfig("kimi_k2", 5, 384, 8, 7168, 2048,
                           (1, 32, 1024, 16384), "zipf", True),
}


def _key(seed: int, tensor: int, expert: int = 0) -> int:
    """A 63-bit draw key from (seed, tensor, expert) (SplitMix64 finaliser)."""
    z = (seed * 0x9E3779B97F4A7C15 + tensor * 0xBF58476D1CE4E5B9
         + (expert + 1) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    return (z ^ (z >> 31)) & 0x7FFFFFFFFFFFFFFF


def _normal(shape, std: float, key: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(key)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def expert_weights_bf16(cfg: LayerConfig, expert: int, which: str,
                        device="cpu") -> torch.Tensor:
    """bf16 N(0, 0.02) weight of one expert linear.

    which = "gate_up" -> [2I, H] (rows [0, I) gate, rows [I, 2I) up)
    which = "down"    -> [H, I]
    """
    if which == "gate_up":
        shape, tid = (2 * cfg.I, cfg.H), _T_GATE_UP
    elif which == "down":
        shape, tid = (cfg.H, cfg.I), _T_DOWN
    else:
        raise ValueError(which)
    return _normal(shape, 0.02, _key(cfg.seed, tid, expert), device).to(torch.bfloat16)


def all_expert_weights_bf16(cfg: LayerConfig, which: str, device="cpu",
                            experts: Optional[Sequence[int]] = None) -> torch.Tensor:
    ids = range(cfg.E) if experts is None else experts
    return torch.stack([expert_weights_bf16(cfg, e, which, device) for e in ids])


def layer_input_bf16(cfg: LayerConfig, T: int, device="cpu") -> torch.Tensor:
    """bf16 [T, H] layer input, N(0, 1) with optional x20 outlier channels."""
    x = _normal((T, cfg.H), 1.0, _key(cfg.seed, _T_X, T), device)
    if cfg.outlier_channels > 0:
        n_out = max(1, int(round(cfg.outlier_channels * cfg.H)))
        rng = np.random.default_rng(_key(cfg.seed, _T_OUTLIER))
        ch = torch.as_tensor(np.sort(rng.choice(cfg.H, n_out, replace=False)), device=device)
        x[:, ch] *= 20.0
    return x.to(torch.bfloat16)


def router_logits(cfg: LayerConfig, T: int, device="cpu") -> torch.Tensor:
    """fp32 [T, E] router logits (N(0,1), plus the Zipf popularity bias)."""
    logits = _normal((T, cfg.E), 1.0, _key(cfg.seed, _T_LOGITS, T), device)
    if cfg.routing == "zipf":
        rng = np.random.default_rng(_key(cfg.seed, _T_BIAS))
        perm = rng.permutation(cfg.E)
        rank = np.empty(cfg.E, dtype=np.float64)
        rank[perm] = np.arange(1, cfg.E + 1, dtype=np.float64)
        p = rank ** -1.1
        p /= p.sum()
        logits = logits + torch.as_tensor(np.log(p), dtype=torch.float32, device=device)
    elif cfg.routing != "uniform":
        raise ValueError(cfg.routing)
    return logits


def route(logits: torch.Tensor, k: int):
    """Softmax router with top-k and renormalised weights (input generator).

    Returns topk_ids int32 [T, k] (descending probability, ties to the lower
    expert id) and topk_w fp32 [T, k] summing to 1 per row.
    """
    p = torch.softmax(logits.float(), dim=-1)
    E = p.shape[-1]
    # ties to the lower id: sort on (-p, id) via a stable sort of -p
    order = torch.sort(-p, dim=-1, stable=True).indices[:, :k]
    w = torch.gather(p, 1, order)
    w = w / w.sum(dim=-1, keepdim=True)
    assert int(order.max()) < E
    return order.to(torch.int32).contiguous(), w.float().contiguous()


def routing(cfg: LayerConfig, T: int, device="cpu"):
    return route(router_logits(cfg, T, device), cfg.k)


def activation_global_scale_input(x: torch.Tensor) -> float:
    """Static per-tensor activation global for gate_up: amax(|x|) / (6 * 448).

    The model cards store an FP32 per-tensor input global scale per expert
    linear ("Compression details" table); the calibration that produced them
    is not given, so the synthetic layer uses the batch amax mapped onto the
    largest representable NVFP4 value (6) times the largest E4M3 scale (448).
    """
    amax = float(x.float().abs().max())
    return float(np.float32(np.float32(amax) / np.float32(2688.0)))
