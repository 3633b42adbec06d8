"""Expert parallelism for the routed-expert MLP: the experts of a layer are split
over the ranks of a process group, each rank holding a contiguous range, and every
rank routes its own tokens (the DP+EP serving layout of the Qwen3.5-397B-A17B-
P48NVFP4-MoESQ model card's serving section).  One exchange each way:

- dispatch: every routed slot's NVFP4 codes and scales go to the rank that holds its
  expert (an all-to-all of 0.53 bytes per element instead of bf16's 2), quantised on
  the token's rank with the expert's input global;
- combine: the bf16 down outputs come back in the same order, and the weighted sum runs
  on the token's rank in j order, as on one GPU.

Because the slot order is (expert, token, j) and each rank's experts are contiguous,
the slots leave already grouped by destination rank; the receiving rank puts them in
its own expert order with a second permutation (k = 1) and a gather into the GEMM's
padded operand layout.  With one rank the result equals the single-GPU forward bit
for bit.

The exchange runs through ``torch.distributed.all_to_all_single`` (NCCL on GPUs).  The
compute is a separate object so that the exchange logic can run on any backend; the
default, ``DeviceCompute``, is the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def expert_ranges(E: int, world: int):
    """Contiguous expert range [lo, hi) of every rank."""
    b = [r * E // world for r in range(world + 1)]
    return [(b[r], b[r + 1]) for r in range(world)]


class DeviceCompute:
    """The steps of the expert-parallel forward on this rank's GPU, with the library's kernels.

    ``local``: MoELayer of this rank's experts (its g_in globals are those experts');
    ``g_in_gate_up_all``: device f32 [E], every expert's gate_up input global (the token's
    rank quantises each slot with the global of the expert that will use it)."""

    def __init__(self, local, g_in_gate_up_all: torch.Tensor):
        from . import _lib as L
        from .layer import EPI_BF16, EPI_SWIGLU_NVFP4, SF_LINEAR
        self.L, self.local = L, local
        self.epi_swiglu, self.epi_bf16, self.sf_linear = EPI_SWIGLU_NVFP4, EPI_BF16, SF_LINEAR
        self.g_all = g_in_gate_up_all.float().contiguous()
        self.dev = self.g_all.device
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def _permute(self, ids, T, k, E):
        i32 = dict(dtype=torch.int32, device=self.dev)
        eo, po = torch.empty(E + 1, **i32), torch.empty(E + 1, **i32)
        st, ts = torch.empty(T * k, **i32), torch.empty(T * k, **i32)
        n = self.L.permute_workspace_size(T, k, E)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=self.dev)
        self.L.moesq_permute(ids.to(torch.int32).contiguous(), T, k, E, eo, po, st, ts, ws, n, self.status)
        return eo, po, st, ts

    def route(self, topk_ids, E):
        """Global permutation of this rank's tokens: (expert_offsets [E+1], slot_token, token_slot)."""
        T, k = topk_ids.shape
        eo, _, st, ts = self._permute(topk_ids, T, k, E)
        return eo, st, ts

    def quantise(self, x, slot_token, expert_offsets, E):
        """NVFP4 codes [S, H/2] and linear scales [S, H/32] of every slot, in slot order."""
        S, H = slot_token.numel(), x.shape[1]
        codes = torch.empty((S, H // 2), dtype=torch.uint8, device=self.dev)
        sf = torch.empty((S, H // 32), dtype=torch.uint8, device=self.dev)
        if S:
            self.L.moesq_quant_act(x.view(torch.uint16), H, slot_token, expert_offsets, None, E, self.g_all, S,
                                   self.sf_linear, codes, sf)
        return codes, sf

    def experts(self, codes, sf, local_ids):
        """This rank's expert MLP on received slots (local expert ids) -> y bf16 [n, H], received order."""
        lay = self.local
        n, H, I, E = codes.shape[0], lay.H, lay.I, lay.E
        y_recv = torch.empty((n, H), dtype=torch.bfloat16, device=self.dev)
        if n == 0:
            return y_recv
        eo, po, st, ts = self._permute(local_ids.view(n, 1), n, 1, E)
        P = self.L.padded_rows(n, E)
        u8 = dict(dtype=torch.uint8, device=self.dev)
        a_codes, a_sf = torch.empty((P, H // 2), **u8), torch.empty((P // 128) * (H // 128) * 512, **u8)
        self.L.moesq_gather_act(codes, sf, st, n, H, eo, po, E, a_codes, a_sf)
        h_codes, h_sf = torch.empty((P, I // 2), **u8), torch.empty((P // 128) * (I // 128) * 512, **u8)
        self.L.moesq_grouped_gemm(lay.gate_up.struct, a_codes, a_sf, lay.g_in_gate_up, eo, po, n, P,
                                  self.epi_swiglu, lay.g_in_down, h_codes, h_sf, d_status=self.status)
        y = torch.empty((n, H), dtype=torch.bfloat16, device=self.dev)
        self.L.moesq_grouped_gemm(lay.down.struct, h_codes, h_sf, lay.g_in_down, eo, po, n, P, self.epi_bf16, None,
                                  y.view(torch.uint16), None, d_status=self.status)
        # back to the received order: a one-slot combine with weight 1 is an exact row gather
        ones = torch.ones(n, dtype=torch.float32, device=self.dev)
        self.L.moesq_unpermute(y.view(torch.uint16), ts, ones, n, 1, H, y_recv.view(torch.uint16))
        return y_recv

    def combine(self, y, token_slot, topk_w):
        T, k = topk_w.shape
        out = torch.empty((T, y.shape[1]), dtype=torch.bfloat16, device=self.dev)
        if T:
            self.L.moesq_unpermute(y.view(torch.uint16), token_slot, topk_w.float().contiguous(), T, k, y.shape[1],
                                   out.view(torch.uint16))
        return out


class ExpertParallelMoE:
    """forward(x [T, H] bf16, topk_ids [T, k] global expert ids, topk_w [T, k]) on every rank
    of ``group`` (all ranks call it, each with its own tokens; T may differ and be 0)."""

    def __init__(self, E: int, k: int, H: int, compute, group=None):
        self.E, self.k, self.H = E, k, H
        self.compute, self.group = compute, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.ranges = expert_ranges(E, self.world)

    def _exchange(self, t: torch.Tensor, send_rows, recv_rows):
        # rows travel as 32-bit words (every row here is a multiple of 4 bytes: NVFP4 codes
        # and scales of K % 128 == 0, bf16 rows of even H, int32 ids), bit-exact on every backend
        t = t.contiguous()
        v = t.view(t.shape[0], -1).view(torch.int32)
        out = torch.empty((sum(recv_rows), v.shape[1]), dtype=torch.int32, device=v.device)
        dist.all_to_all_single(out, v, output_split_sizes=list(recv_rows), input_split_sizes=list(send_rows),
                               group=self.group)
        return out.view(t.dtype).view((sum(recv_rows),) + tuple(t.shape[1:]))

    def forward(self, x, topk_ids, topk_w):
        c = self.compute
        eo, slot_token, token_slot = c.route(topk_ids, self.E)
        codes, sf = c.quantise(x, slot_token, eo, self.E)
        eo_h = eo.cpu().tolist()
        send = [eo_h[hi] - eo_h[lo] for lo, hi in self.ranges]
        # the counts travel on the payload's device (NCCL moves device tensors only)
        recv_t = torch.empty(self.world, dtype=torch.int64, device=codes.device)
        dist.all_to_all_single(recv_t, torch.tensor(send, dtype=torch.int64, device=codes.device), group=self.group)
        recv = recv_t.cpu().tolist()
        # local expert id of every slot, in slot order (slots are grouped by rank already),
        # built where the slots live
        dv = codes.device
        counts = (eo[1:] - eo[:-1]).to(torch.int64)
        e_of_slot = torch.repeat_interleave(torch.arange(self.E, dtype=torch.int64, device=dv), counts.to(dv),
                                            output_size=int(eo_h[-1]))
        bounds = torch.tensor([hi for _, hi in self.ranges], dtype=torch.int64, device=dv)
        lows = torch.tensor([lo for lo, _ in self.ranges], dtype=torch.int64, device=dv)
        local_ids = (e_of_slot - lows[torch.bucketize(e_of_slot, bounds, right=True)]).to(torch.int32)
        r_codes = self._exchange(codes, send, recv)
        r_sf = self._exchange(sf, send, recv)
        r_ids = self._exchange(local_ids, send, recv)
        y_recv = c.experts(r_codes, r_sf, r_ids)
        y = self._exchange(y_recv, recv, send)
        return c.combine(y, token_slot, topk_w)
