"""Device-resident expert weights and the MoE expert layer (user-facing helpers).

These classes own torch CUDA buffers and call the C ABI; they do no arithmetic
of their own.  Typical use:

    st  = quantize_expert_weights(w_gate_up_bf16, n_seg=2)        # export (prune+quant+encode)
    gu  = ExpertLinear.from_storage(st, kind=KIND_GATE_UP_SPLIT)   # load-time repack
    dn  = ExpertLinear.from_storage(quantize_expert_weights(w_down_bf16), kind=KIND_DOWN)
    moe = MoELayer(k, gu, dn, g_in_gate_up, g_in_down)
    out = moe.forward(x_bf16, topk_ids, topk_w)
"""
from __future__ import annotations

import torch

from . import _lib as L

KIND_DOWN, KIND_GATE_UP, KIND_GATE_UP_SPLIT, KIND_GATE_UP_EXACT = 0, 1, 2, 3
EPI_F32, EPI_BF16, EPI_SWIGLU_NVFP4 = 0, 1, 2
SF_LINEAR, SF_KERNEL = 0, 1


def _u16(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint16) if t.dtype == torch.bfloat16 else t


def quantize_expert_weights(w: torch.Tensor, n_seg: int = 1, stream=None) -> dict:
    """bf16 CUDA weights [E, out, K] -> pair-bitmask storage on the same device."""
    assert w.is_cuda and w.dtype == torch.bfloat16 and w.dim() == 3
    w = w.contiguous()
    E, out, K = w.shape
    dev = w.device
    packed = torch.empty((E, out, K // 4), dtype=torch.uint8, device=dev)
    mask = torch.empty((E, out, K // 16), dtype=torch.uint8, device=dev)
    scale = torch.empty((E, out, K // 32), dtype=torch.uint8, device=dev)
    g_w = torch.empty((E, n_seg), dtype=torch.float32, device=dev)
    ws_bytes = L.quant_weight_workspace_size(E, n_seg)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    L.moesq_quant_weight(_u16(w), E, out, K, n_seg, packed, mask, scale, g_w, ws, ws_bytes, stream)
    return dict(packed=packed, mask=mask, scale=scale, g_w=g_w, E=E, out=out, K=K)


class ExpertLinear:
    """One expert linear over all experts in the GEMM's operand layouts."""

    def __init__(self, packed, meta, sf, alpha_w, E, out, K, kind):
        self.packed, self.meta, self.sf, self.alpha_w = packed, meta, sf, alpha_w
        self.E, self.out, self.K, self.kind = E, out, K, kind
        self.struct = L.Linear(packed.data_ptr(), meta.data_ptr(), sf.data_ptr(), alpha_w.data_ptr(),
                               out, K, E, kind)

    @classmethod
    def from_storage(cls, st: dict, kind: int, d_status=None, stream=None) -> "ExpertLinear":
        E, out, K = st["E"], st["out"], st["K"]
        dev = st["packed"].device
        mb, sb = L.repack_sizes(out, K)
        meta = torch.empty(E * mb, dtype=torch.uint8, device=dev)
        sf = torch.empty(E * sb, dtype=torch.uint8, device=dev)
        alpha = torch.empty(2 * E if kind == KIND_GATE_UP_EXACT else E, dtype=torch.float32, device=dev)
        L.moesq_repack_meta(st["mask"], st["scale"], st["g_w"].contiguous(), E, out, K, kind, meta, sf,
                            alpha, d_status, stream)
        return cls(st["packed"], meta, sf, alpha, E, out, K, kind)


class MoELayer:
    """The routed-expert MLP of one MoE layer on one GPU."""

    def __init__(self, k: int, gate_up: ExpertLinear, down: ExpertLinear, g_in_gate_up: torch.Tensor,
                 g_in_down: torch.Tensor):
        assert gate_up.E == down.E and gate_up.out == 2 * down.K and gate_up.K == down.out
        self.E, self.k, self.H, self.I = gate_up.E, k, gate_up.K, down.K
        self.gate_up, self.down = gate_up, down
        self.g_in_gate_up = g_in_gate_up.float().contiguous()
        self.g_in_down = g_in_down.float().contiguous()
        self.struct = L.MoeLayer(self.E, k, self.H, self.I, gate_up.struct, down.struct,
                                 self.g_in_gate_up.data_ptr(), self.g_in_down.data_ptr())
        self._ws = None

    def workspace(self, T: int, host: bool = False) -> torch.Tensor:
        n = (L.moe_forward_host_workspace_size if host else L.moe_forward_workspace_size)(self.struct, T)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.gate_up.packed.device)
        return self._ws

    def forward(self, x, topk_ids, topk_w, out=None, d_status=None, stream=None):
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        ws = self.workspace(T)
        L.moesq_moe_forward(self.struct, _u16(x), topk_ids, topk_w, T, _u16(out), ws, ws.numel(),
                            d_status, stream)
        return out

    def forward_host(self, h_x, h_ids, h_w, h_out, d_status=None, stream=None):
        """Host (ideally pinned) buffers in and out; synchronises the stream."""
        T = h_x.shape[0]
        ws = self.workspace(T, host=True)
        L.moesq_moe_forward_host(self.struct, _u16(h_x), h_ids, h_w, T, _u16(h_out), ws, ws.numel(),
                                 d_status, stream)
        return h_out
