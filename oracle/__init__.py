"""CPU oracle for the paired-4:8 sparse NVFP4 MoE expert path -- TEST INFRASTRUCTURE.

A plain, slow, float64/int64 restatement of what the path computes, written
from the MoESQ pages (model cards of Qwen3.5-397B-A17B-, Qwen3.8-Flash-Next-
and Qwen3-30B-A3B-P48NVFP4-MoESQ, and the MoESQ repository README).  It shares
no code with the CUDA library and imports nothing from it.  Only the tests,
the smoke check and the CPU-baseline leg of the benchmark may use it; the
product path never does.

Modules:
  formats  -- E2M1, E4M3 and bf16 rounding from their format definitions
  nvfp4    -- per-32 block-scaled NVFP4 quantisation rule
  storage  -- paired-4:8 pruning, pair-bitmask encode/decode, gate/up fold,
              the tensor-core metadata and scale-factor layouts
  routing  -- stable expert permutation and the weighted combine
  gemm     -- exact grouped GEMMs, SwiGLU, the whole expert MLP

Every function here is pinned by a "not gpu" test against values the pages or
mathematics fix (tests/test_oracle_*.py).
"""
from . import formats, gemm, nvfp4, routing, storage  # noqa: F401
