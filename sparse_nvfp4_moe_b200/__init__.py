"""sparse_nvfp4_moe_b200 -- paired-4:8 sparse NVFP4 MoE expert GEMMs on B200 (sm_100a).

The compute lives in libmoesq.so (hand-written CUDA for sm_100a behind the C ABI
of include/moesq.h).  This package is a thin ctypes binding with the same entry
point names plus small helpers that own device buffers; torch provides device
memory and streams.  There is no CPU or library fallback: calls raise if the
shared library is missing.
"""
from ._lib import (Linear, MoeLayer, MoesqError, declared_symbols, lib, moesq_decode,  # noqa: F401
                   moesq_encode, moesq_gather_act, moesq_gemm_launch_pairs, moesq_set_gemm_pair_limit,
                   moesq_gemm_tiles_per_item, moesq_set_gemm_tiles_per_item, moesq_measure_sparse_mma_peak,
                   moesq_grouped_gemm, moesq_grouped_gemm_dense,
                   moesq_grouped_gemm_down_combine, moesq_moe_forward,
                   moesq_moe_forward_host, moesq_selftest_wait_timeout, moesq_sf_expand_block16,
                   moesq_permute, moesq_permute_noalloc, moesq_quant_act, moesq_quant_act_routed, moesq_quant_weight, moesq_repack_meta,
                   moesq_unpermute, moe_forward_host_workspace_size, moe_forward_workspace_size,
                   padded_rows, permute_workspace_size, quant_weight_workspace_size, repack_sizes,
                   status_string)
from .layer import (EPI_BF16, EPI_F32, EPI_SWIGLU_NVFP4, KIND_DOWN, KIND_GATE_UP,  # noqa: F401
                    KIND_GATE_UP_EXACT, KIND_GATE_UP_SPLIT, SF_KERNEL, SF_LINEAR, ExpertLinear, MoELayer,
                    quantize_expert_weights)

__all__ = [n for n in dir() if not n.startswith("_")]
