"""ctypes binding of libmoesq.so: argument marshalling only, no arithmetic.

Every public function mirrors a C entry point of include/moesq.h with the same
name.  Tensors are torch CUDA tensors (torch is used for device memory and
streams only); their data pointers and the current CUDA stream are passed to
the library.  A missing or unloadable library raises at import of the first
call: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoesq.so")

c_i32, c_i64, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class MoesqError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: status {status} ({text})")
        self.status = status


class Linear(ctypes.Structure):
    _fields_ = [("packed", c_vp), ("meta", c_vp), ("sf", c_vp), ("alpha_w", c_vp),
                ("out", c_i64), ("K", c_i64), ("E", c_i32), ("kind", c_i32)]


class MoeLayer(ctypes.Structure):
    _fields_ = [("E", c_i32), ("k", c_i32), ("H", c_i64), ("I", c_i64),
                ("gate_up", Linear), ("down", Linear),
                ("g_in_gate_up", c_vp), ("g_in_down", c_vp)]


_SIGS = {
    "moesq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moesq_abi_version": (ctypes.c_int, []),
    "moesq_decode": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp]),
    "moesq_encode": (ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp]),
    "moesq_quant_weight": (ctypes.c_int, [c_vp, c_i64, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp, c_vp,
                                          c_vp, c_sz, c_vp]),
    "moesq_quant_weight_workspace_size": (ctypes.c_int, [c_i64, c_i32, ctypes.POINTER(c_sz)]),
    "moesq_repack_sizes": (ctypes.c_int, [c_i64, c_i64, ctypes.POINTER(c_sz), ctypes.POINTER(c_sz)]),
    "moesq_repack_meta": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i32, c_vp, c_vp,
                                         c_vp, c_vp, c_vp]),
    "moesq_permute": (ctypes.c_int, [c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz,
                                     c_vp, c_vp]),
    "moesq_permute_workspace_size": (ctypes.c_int, [c_i64, c_i32, c_i32, ctypes.POINTER(c_sz)]),
    "moesq_permute_noalloc": (ctypes.c_int, [c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "moesq_padded_rows": (c_i64, [c_i64, c_i32]),
    "moesq_unpermute": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i32, c_i64, c_vp, c_vp]),
    "moesq_quant_act": (ctypes.c_int, [c_vp, c_i64, c_vp, c_vp, c_vp, c_i32, c_vp, c_i64, c_i32, c_vp,
                                       c_vp, c_vp]),
    "moesq_quant_act_routed": (ctypes.c_int, [c_vp, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_i32,
                                              c_vp, c_vp, c_vp, c_vp]),
    "moesq_grouped_gemm": (ctypes.c_int, [ctypes.POINTER(Linear), c_vp, c_vp, c_vp, c_vp, c_vp, c_i64,
                                          c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp]),
    "moesq_grouped_gemm_down_combine": (ctypes.c_int, [ctypes.POINTER(Linear), c_vp, c_vp, c_vp, c_vp, c_vp, c_i64,
                                                       c_i64, c_vp, c_vp, c_vp, c_i64, c_i32, c_vp, c_vp, c_vp,
                                                       c_vp, c_vp]),
    "moesq_grouped_gemm_dense": (ctypes.c_int, [ctypes.POINTER(Linear), c_vp, c_vp, c_vp, c_vp, c_vp, c_i64,
                                                c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "moesq_sf_expand_block16": (ctypes.c_int, [c_vp, c_vp, c_i64, c_vp]),
    "moesq_set_gemm_pair_limit": (ctypes.c_int, [c_i32]),
    "moesq_gemm_launch_pairs": (ctypes.c_int, [c_i32, c_i32, ctypes.POINTER(c_i32)]),
    "moesq_set_gemm_tiles_per_item": (ctypes.c_int, [c_i32]),
    "moesq_measure_sparse_mma_peak": (ctypes.c_int, [c_i32, c_i32, ctypes.POINTER(ctypes.c_double), c_vp, c_vp]),
    "moesq_gemm_tiles_per_item": (ctypes.c_int, [c_i32, c_i32, c_i64, c_i64, c_i64, ctypes.POINTER(c_i32)]),
    "moesq_selftest_wait_timeout": (ctypes.c_int, [c_vp, c_i64, c_vp, c_vp]),
    "moesq_gather_act": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp]),
    "moesq_grouped_gemm_workspace_size": (ctypes.c_int, [ctypes.POINTER(Linear), c_i64,
                                                         ctypes.POINTER(c_sz)]),
    "moesq_moe_forward": (ctypes.c_int, [ctypes.POINTER(MoeLayer), c_vp, c_vp, c_vp, c_i64, c_vp, c_vp,
                                         c_sz, c_vp, c_vp]),
    "moesq_moe_forward_workspace_size": (ctypes.c_int, [ctypes.POINTER(MoeLayer), c_i64,
                                                        ctypes.POINTER(c_sz)]),
    "moesq_moe_forward_host": (ctypes.c_int, [ctypes.POINTER(MoeLayer), c_vp, c_vp, c_vp, c_i64, c_vp,
                                              c_vp, c_sz, c_vp, c_vp]),
    "moesq_moe_forward_host_workspace_size": (ctypes.c_int, [ctypes.POINTER(MoeLayer), c_i64,
                                                             ctypes.POINTER(c_sz)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was not built (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_nvfp4_moe_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def declared_symbols():
    return sorted(_SIGS)


def _check(fn: str, st: int):
    if st != 0:
        raise MoesqError(fn, st, lib().moesq_status_string(st).decode())


def _p(t):
    """Data pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(code: int) -> str:
    return lib().moesq_status_string(code).decode()


# -------------------------------------------------------------- size queries --

def _size_out(fn, *args):
    n = c_sz(0)
    _check(fn, getattr(lib(), fn)(*args, ctypes.byref(n)))
    return n.value


def quant_weight_workspace_size(E, n_seg):
    return _size_out("moesq_quant_weight_workspace_size", E, n_seg)


def permute_workspace_size(T, k, E):
    return _size_out("moesq_permute_workspace_size", T, k, E)


def repack_sizes(out, K):
    a, b = c_sz(0), c_sz(0)
    _check("moesq_repack_sizes", lib().moesq_repack_sizes(out, K, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def padded_rows(S, E):
    return int(lib().moesq_padded_rows(S, E))


def moe_forward_workspace_size(layer: MoeLayer, T):
    return _size_out("moesq_moe_forward_workspace_size", ctypes.byref(layer), T)


def moe_forward_host_workspace_size(layer: MoeLayer, T):
    return _size_out("moesq_moe_forward_host_workspace_size", ctypes.byref(layer), T)


# ------------------------------------------------------------------ entries --

def moesq_decode(packed, mask, dense, rows, K, d_status=None, stream=None):
    _check("moesq_decode", lib().moesq_decode(_p(packed), _p(mask), _p(dense), rows, K,
                                              _p(d_status), _stream(stream)))


def moesq_encode(dense, mask_hint, packed, mask, rows, K, d_status=None, stream=None):
    _check("moesq_encode", lib().moesq_encode(_p(dense), _p(mask_hint), _p(packed), _p(mask), rows, K,
                                              _p(d_status), _stream(stream)))


def moesq_quant_weight(w, E, out, K, n_seg, packed, mask, scale, g_w, ws, ws_bytes, stream=None):
    _check("moesq_quant_weight", lib().moesq_quant_weight(_p(w), E, out, K, n_seg, _p(packed), _p(mask),
                                                          _p(scale), _p(g_w), _p(ws), ws_bytes,
                                                          _stream(stream)))


def moesq_repack_meta(mask, scale, g_w, E, out, K, kind, meta, sf, alpha_w, d_status=None, stream=None):
    _check("moesq_repack_meta", lib().moesq_repack_meta(_p(mask), _p(scale), _p(g_w), E, out, K, kind,
                                                        _p(meta), _p(sf), _p(alpha_w), _p(d_status),
                                                        _stream(stream)))


def moesq_permute(topk_ids, T, k, E, expert_offsets, pad_offsets, slot_token, token_slot, ws, ws_bytes,
                  d_status=None, stream=None):
    _check("moesq_permute", lib().moesq_permute(_p(topk_ids), T, k, E, _p(expert_offsets),
                                                _p(pad_offsets), _p(slot_token), _p(token_slot),
                                                _p(ws), ws_bytes, _p(d_status), _stream(stream)))


def moesq_permute_noalloc(topk_ids, T, k, E, expert_offsets, pad_offsets, slot_token, token_slot,
                          d_status=None, stream=None):
    """moesq_permute without a workspace argument (fixed device scratch; see the header)."""
    _check("moesq_permute_noalloc", lib().moesq_permute_noalloc(
        _p(topk_ids), T, k, E, _p(expert_offsets), _p(pad_offsets), _p(slot_token), _p(token_slot),
        _p(d_status), _stream(stream)))


PERMUTE_NOALLOC_MAX_COUNTS = 262144


def moesq_unpermute(y, token_slot, topk_w, T, k, H, out, stream=None):
    _check("moesq_unpermute", lib().moesq_unpermute(_p(y), _p(token_slot), _p(topk_w), T, k, H, _p(out),
                                                    _stream(stream)))


def moesq_quant_act(x, K, gather, expert_offsets, pad_offsets, E, g_in, rows, layout, codes, sf,
                    stream=None):
    _check("moesq_quant_act", lib().moesq_quant_act(_p(x), K, _p(gather), _p(expert_offsets),
                                                    _p(pad_offsets), E, _p(g_in), rows, layout,
                                                    _p(codes), _p(sf), _stream(stream)))


def moesq_quant_act_routed(x, T, K, topk_ids, token_slot, k, expert_offsets, pad_offsets, E, g_in, codes,
                           sf, stream=None):
    _check("moesq_quant_act_routed", lib().moesq_quant_act_routed(
        _p(x), T, K, _p(topk_ids), _p(token_slot), k, _p(expert_offsets), _p(pad_offsets), E, _p(g_in),
        _p(codes), _p(sf), _stream(stream)))


def moesq_grouped_gemm(W: Linear, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap,
                       epilogue, g_next, out, out_sf, ws=None, ws_bytes=0, d_status=None, stream=None):
    _check("moesq_grouped_gemm", lib().moesq_grouped_gemm(
        ctypes.byref(W), _p(act_codes), _p(act_sf), _p(g_act), _p(expert_offsets), _p(pad_offsets), S,
        P_cap, epilogue, _p(g_next), _p(out), _p(out_sf), _p(ws), ws_bytes, _p(d_status),
        _stream(stream)))


def moesq_grouped_gemm_down_combine(W: Linear, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap,
                                    slot_token, token_slot, topk_w, T, k, y, out, arrivals, d_status=None,
                                    stream=None):
    _check("moesq_grouped_gemm_down_combine", lib().moesq_grouped_gemm_down_combine(
        ctypes.byref(W), _p(act_codes), _p(act_sf), _p(g_act), _p(expert_offsets), _p(pad_offsets), S, P_cap,
        _p(slot_token), _p(token_slot), _p(topk_w), T, k, _p(y), _p(out), _p(arrivals), _p(d_status),
        _stream(stream)))


def moesq_grouped_gemm_dense(W: Linear, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap,
                             epilogue, g_next, out, out_sf, d_status=None, stream=None):
    _check("moesq_grouped_gemm_dense", lib().moesq_grouped_gemm_dense(
        ctypes.byref(W), _p(act_codes), _p(act_sf), _p(g_act), _p(expert_offsets), _p(pad_offsets), S,
        P_cap, epilogue, _p(g_next), _p(out), _p(out_sf), _p(d_status), _stream(stream)))


def moesq_gather_act(codes_in, sf_in, gather, S, K, expert_offsets, pad_offsets, E, codes_out, sf_out,
                     stream=None):
    _check("moesq_gather_act", lib().moesq_gather_act(_p(codes_in), _p(sf_in), _p(gather), S, K, _p(expert_offsets),
                                                      _p(pad_offsets), E, _p(codes_out), _p(sf_out),
                                                      _stream(stream)))


def moesq_selftest_wait_timeout(d_status, limit_ns, d_gave_up, stream=None):
    _check("moesq_selftest_wait_timeout", lib().moesq_selftest_wait_timeout(_p(d_status), limit_ns, _p(d_gave_up),
                                                                              _stream(stream)))


def moesq_sf_expand_block16(sf32, sf16, nblocks, stream=None):
    _check("moesq_sf_expand_block16", lib().moesq_sf_expand_block16(_p(sf32), _p(sf16), nblocks, _stream(stream)))


def moesq_moe_forward(layer: MoeLayer, x, topk_ids, topk_w, T, out, ws, ws_bytes, d_status=None,
                      stream=None):
    _check("moesq_moe_forward", lib().moesq_moe_forward(ctypes.byref(layer), _p(x), _p(topk_ids),
                                                        _p(topk_w), T, _p(out), _p(ws), ws_bytes,
                                                        _p(d_status), _stream(stream)))


def moesq_moe_forward_host(layer: MoeLayer, h_x, h_topk_ids, h_topk_w, T, h_out, ws, ws_bytes,
                           d_status=None, stream=None):
    _check("moesq_moe_forward_host", lib().moesq_moe_forward_host(
        ctypes.byref(layer), _p(h_x), _p(h_topk_ids), _p(h_topk_w), T, _p(h_out), _p(ws), ws_bytes,
        _p(d_status), _stream(stream)))


def moesq_set_gemm_pair_limit(max_pairs):
    _check("moesq_set_gemm_pair_limit", lib().moesq_set_gemm_pair_limit(max_pairs))


def moesq_gemm_launch_pairs(dense, epilogue):
    """CTA pairs the next grouped-GEMM launch on the current device would use."""
    n = c_i32(0)
    _check("moesq_gemm_launch_pairs", lib().moesq_gemm_launch_pairs(dense, epilogue, ctypes.byref(n)))
    return n.value


def moesq_measure_sparse_mma_peak(iters=2000, n=256, d_status=None, stream=None):
    """Dense-equivalent TFLOP/s of back-to-back sparse FP4 MMAs on every CTA pair (synchronises)."""
    v = ctypes.c_double(0.0)
    _check("moesq_measure_sparse_mma_peak",
           lib().moesq_measure_sparse_mma_peak(iters, n, ctypes.byref(v), _p(d_status), _stream(stream)))
    return v.value


def moesq_set_gemm_tiles_per_item(tiles):
    _check("moesq_set_gemm_tiles_per_item", lib().moesq_set_gemm_tiles_per_item(tiles))


def moesq_gemm_tiles_per_item(dense, epilogue, K, E, S):
    """Token tiles per work item (1, or 2 for wide items) a grouped-GEMM launch would use."""
    n = c_i32(0)
    _check("moesq_gemm_tiles_per_item", lib().moesq_gemm_tiles_per_item(dense, epilogue, K, E, S, ctypes.byref(n)))
    return n.value
