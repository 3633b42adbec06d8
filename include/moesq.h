/*
 * moesq.h -- C ABI of the paired-4:8 sparse NVFP4 MoE expert library (sm_100a).
 *
 * The library runs the routed-expert MLP of a Mixture-of-Experts layer whose
 * expert weights are NVFP4 (E2M1) with paired-4:8 structured sparsity along K,
 * an FP8-E4M3 block scale per 32 dense K elements and an FP32 per-tensor global
 * scale, kept in "pair-bitmask" storage; activations are NVFP4 with dynamic
 * per-32 group scales and a static FP32 global per expert linear.  Sources:
 *   [storage]  "Sparse storage layout (paired48_sparse, pair-bitmask v1)",
 *              Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card;
 *   [format]   "Compression details" table, same card;
 *   [kernel]   header list of the same card (paired-4:8 sparse NVFP4 grouped
 *              GEMM, SM100) and the MoESQ repository README ("Kernels");
 *   [fold]     gate/up global-scale note of the Qwen3.8-Flash-Next- and
 *              Qwen3-30B-A3B-P48NVFP4-MoESQ model cards;
 *   [export]   MoESQ repository README, "Usage" (Output bullet).
 *
 * Conventions common to every call
 *  - Pointers named d_* or documented as "device" are CUDA device pointers; the
 *    caller owns every buffer.  No call allocates, frees or synchronises, except
 *    moesq_moe_forward_host (host buffers, internal copy streams; documented there).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream);
 *    work is enqueued asynchronously on it.
 *  - Row-major, K innermost.  A packed NVFP4 byte holds element 2i in its low
 *    nibble and element 2i+1 in its high nibble.  bf16 tensors are passed as
 *    uint16_t bit patterns.
 *  - Argument errors (null pointers, bad sizes, misalignment, too-small
 *    workspace) are returned synchronously and nothing is enqueued.
 *    Data-dependent errors found on the device (bad mask nibble, expert id out
 *    of range, a bounded wait that gave up) are OR-ed as MOESQ_DFLAG_* bits into
 *    the caller's int32 word `d_status` (device memory, may be NULL to ignore);
 *    the caller reads it when it chooses.  A flagged call still writes only
 *    inside its output buffers.
 *  - Every device pointer must be 16-byte aligned.
 *
 * Arithmetic readings (the pages name the formats, not the arithmetic):
 *  - NVFP4 quantisation of a group of 32 values x with global g (weights and
 *    activations alike), every step IEEE binary32 round-to-nearest-even:
 *        amax = max|x|;  s = amax / (6*g) (s = 0 if 6*g == 0);
 *        sc = E4M3(s), nearest-even, saturating at 448;
 *        sdq = value(sc) * g;  if sdq == 0 all codes are 0x0, else
 *        inv = 1/sdq and code = E2M1(x * inv): nearest of {0,.5,1,1.5,2,3,4,6},
 *        ties to the even code, |v| > 6 -> 6, sign bit = sign of the input.
 *  - Weight global g_w = amax|W_pruned| / (6*448), the multiplier convention.
 *  - Gate/up fold [fold]: the kernel applies the gate global to the fused
 *    gate_up weight; each up block scale sc becomes E4M3(value(sc) * (g_up /
 *    g_gate)) (nearest-even, saturating).
 *  - SwiGLU: h = silu(gate) * up, silu(x) = x / (1 + exp(-x)), gate = rows
 *    [0, I) of the fused [2I, K] weight, up = rows [I, 2I).
 *  - Combine: out[t] = sum_j w[t,j] * y[slot(t,j)], float32 in j order (one
 *    rounding per product and per sum), then bf16 nearest-even.
 */
#ifndef MOESQ_H
#define MOESQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moesq_status {
  MOESQ_OK = 0,
  MOESQ_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum, misaligned pointer */
  MOESQ_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside what the kernels support (see each call) */
  MOESQ_ERR_BAD_SPARSITY = 3,      /* host-visible sparsity violation (moesq_*_host helpers only) */
  MOESQ_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed (launch, tensor map) */
  MOESQ_ERR_TIMEOUT = 5,           /* reserved for callers that translate MOESQ_DFLAG_TIMEOUT */
  MOESQ_ERR_WORKSPACE = 6,         /* workspace pointer NULL or smaller than required */
  MOESQ_ERR_DEVICE = 7,            /* current device is not sm_100 */
  MOESQ_ERR_CAPACITY = 8           /* request larger than the fixed scratch of an
                                      allocation-free entry point */
} moesq_status;

/* bits OR-ed into *d_status by the device */
#define MOESQ_DFLAG_BAD_SPARSITY 0x1 /* a mask nibble without exactly 2 bits set, or
                                        a dense chunk with more than 2 nonzero bytes */
#define MOESQ_DFLAG_BAD_EXPERT 0x2   /* a top-k expert id outside [0, E) */
#define MOESQ_DFLAG_TIMEOUT 0x4      /* a bounded pipeline wait gave up; outputs are garbage */
#define MOESQ_DFLAG_CAPACITY 0x8     /* routed rows exceed the capacity passed by the caller */

typedef void* moesq_stream_t; /* a cudaStream_t */

/* Human-readable text of a status code (static storage). */
const char* moesq_status_string(int status);

/* ABI version of this header (incremented on any incompatible change). */
int moesq_abi_version(void);

/* ------------------------------------------------------------------------- *
 * Storage codecs  [storage], [export]
 * ------------------------------------------------------------------------- */

/* Pair-bitmask -> dense packed NVFP4.
 *   packed  device u8 [rows, K/4]   weight_sparse_packed (2 kept bytes of every 4, K order)
 *   mask    device u8 [rows, K/16]  weight_sparse_mask (bit i = byte i kept, low nibble = lower-K chunk)
 *   dense   device u8 [rows, K/2]   output: kept bytes in place, pruned bytes 0
 * K % 64 == 0.  A nibble without exactly 2 bits set raises MOESQ_DFLAG_BAD_SPARSITY
 * and its chunk is written as zeros.  Lossless: encode(decode(p, m), m) == (p, m). */
moesq_status moesq_decode(const uint8_t* packed, const uint8_t* mask, uint8_t* dense,
                          int64_t rows, int64_t K, int32_t* d_status, moesq_stream_t stream);

/* Dense packed NVFP4 -> pair-bitmask.
 *   dense     device u8 [rows, K/2]
 *   mask_hint device u8 [rows, K/16] or NULL.  With a hint the hinted bytes are kept
 *             (nonzero bytes outside it raise MOESQ_DFLAG_BAD_SPARSITY); without it
 *             the nonzero bytes are kept and each chunk is filled up to 2 with its
 *             lowest-index zero bytes (more than 2 nonzero bytes raises the flag).
 *   packed    device u8 [rows, K/4] output;  mask device u8 [rows, K/16] output
 *             (may alias mask_hint).
 * K % 64 == 0. */
moesq_status moesq_encode(const uint8_t* dense, const uint8_t* mask_hint, uint8_t* packed,
                          uint8_t* mask, int64_t rows, int64_t K, int32_t* d_status,
                          moesq_stream_t stream);

/* Export of bf16 expert weights to pair-bitmask NVFP4 storage (prune + quantise +
 * encode), E experts at once.
 *   w       device bf16 [E, out, K]
 *   n_seg   1 or 2: rows [0,out) split into n_seg equal segments, each with its own
 *           FP32 global (2 = fused gate_up with separate gate and up globals)
 *   packed  device u8 [E, out, K/4];  mask device u8 [E, out, K/16];
 *   scale   device u8 [E, out, K/32] (E4M3 codes);  g_w device f32 [E, n_seg]
 *   ws      device workspace of moesq_quant_weight_workspace_size() bytes
 * Pruning: each 8-element chunk keeps the 2 pairs with the largest a*a+b*b (fp32 on
 * the bf16 values; ties to the lower pair).  Then the NVFP4 rule above with
 * g_w = amax/(6*448) per segment.  K % 64 == 0, out % n_seg == 0. */
moesq_status moesq_quant_weight(const uint16_t* w, int64_t E, int64_t out, int64_t K,
                                int32_t n_seg, uint8_t* packed, uint8_t* mask, uint8_t* scale,
                                float* g_w, void* ws, size_t ws_bytes, moesq_stream_t stream);
moesq_status moesq_quant_weight_workspace_size(int64_t E, int32_t n_seg, size_t* bytes);

/* ------------------------------------------------------------------------- *
 * Load-time repack into the tensor-core operand layouts  [storage] ("at load
 * time ... compresses it into the kernel's own layout"), [fold]
 * ------------------------------------------------------------------------- */

typedef enum moesq_linear_kind {
  MOESQ_LINEAR_DOWN = 0,          /* plain linear [out, K] */
  MOESQ_LINEAR_GATE_UP = 1,       /* fused [2I, K], gate rows first, one global (g_w[e]) */
  MOESQ_LINEAR_GATE_UP_SPLIT = 2, /* fused [2I, K], globals g_w[2e] (gate), g_w[2e+1] (up): the
                                     up/gate ratio is folded into the up block scales (lossy by at
                                     most half an E4M3 step, the pages' load-time fold) */
  MOESQ_LINEAR_GATE_UP_EXACT = 3  /* fused [2I, K], globals g_w[2e] (gate), g_w[2e+1] (up): not
                                     folded; the GEMM applies each global to its own half */
} moesq_linear_kind;

/* Bytes of the repacked metadata and block scales of ONE expert linear. */
moesq_status moesq_repack_sizes(int64_t out, int64_t K, size_t* meta_bytes, size_t* sf_bytes);

/* Mask + block scales -> tcgen05 sparse metadata and scale-factor blocks.
 *   mask   device u8 [E, out, K/16];  scale device u8 [E, out, K/32];
 *   g_w    device f32 [E] (DOWN, GATE_UP) or [E, 2] (GATE_UP_SPLIT, GATE_UP_EXACT)
 *   meta   device u8 [E * meta_bytes]: per expert, per 128-row tile, per 256 dense
 *          K: 128 rows x 16 bytes, row r at 16r; each chunk's nibble = i0 | i1<<2
 *          (ascending kept byte positions), lower-K chunk in the low nibble
 *   sf     device u8 [E * sf_bytes]: per expert, per tile, per 128 dense K a 512-byte
 *          block, row r scale j at (r%32)*16 + (r/32)*4 + j
 *   alpha_w device f32 [E]: the weight global the GEMM applies (gate global for gate_up);
 *          [E, 2] (gate, up) for GATE_UP_EXACT
 * Tile row order: DOWN tile t holds rows 128t..128t+127, tile row 16g + 8p + j being
 * row 128t + 16g + 2j + p (g < 8; p < 2; j < 8); GATE_UP tile t holds the gate and up rows of outputs
 * 64t..64t+63: tile row r = 32q + 16h + 8s + j (q < 4; h, s < 2; j < 8) is source row
 * s*I + 64t + 16q + 2j + h.  The packed values are used as stored (no repack).
 * out % 128 == 0, K % 128 == 0.  Bad nibbles raise MOESQ_DFLAG_BAD_SPARSITY. */
moesq_status moesq_repack_meta(const uint8_t* mask, const uint8_t* scale, const float* g_w,
                               int64_t E, int64_t out, int64_t K, int32_t kind, uint8_t* meta,
                               uint8_t* sf, float* alpha_w, int32_t* d_status,
                               moesq_stream_t stream);

/* ------------------------------------------------------------------------- *
 * Routing  ([kernel]: the grouped GEMM runs over the tokens routed to each expert)
 * ------------------------------------------------------------------------- */

/* Top-k routing -> per-expert contiguous slot groups, order (expert, token, j).
 *   topk_ids      device i32 [T, k]
 *   expert_offsets device i32 [E+1] output: exclusive scan of per-expert counts
 *   pad_offsets   device i32 [E+1] output: same with each count rounded up to 128
 *                 (row of expert e's first slot in the padded activation buffers)
 *   slot_token    device i32 [T*k] output: token of each slot
 *   token_slot    device i32 [T, k] output: slot of each (token, j)
 *   ws            device workspace of moesq_permute_workspace_size() bytes
 * Ids outside [0, E) raise MOESQ_DFLAG_BAD_EXPERT and are routed to expert 0.
 * 1 <= E <= 4096, 1 <= k <= 32, T*k < 2^31. */
moesq_status moesq_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                           int32_t* expert_offsets, int32_t* pad_offsets, int32_t* slot_token,
                           int32_t* token_slot, void* ws, size_t ws_bytes, int32_t* d_status,
                           moesq_stream_t stream);
moesq_status moesq_permute_workspace_size(int64_t T, int32_t k, int32_t E, size_t* bytes);

/* Allocation-free variant of moesq_permute (the pages have no counterpart: this is a
 * library convenience).  Same arguments, outputs and device flags as moesq_permute,
 * minus the workspace: its scratch is a fixed 1 MiB array in device memory that the
 * library declares statically, so it never calls cudaMalloc, cudaFree or any other
 * allocating routine.  It is for callers that cannot allocate device memory when
 * they route a batch -- a serving engine that reserves all device memory up front
 * and forbids later allocations (a late cudaMalloc can fail or stall every stream
 * on the device), or a plugin interface that hands the kernel only its bound input
 * and output buffers.
 *   Limit: ceil(T*k / 1024) * E <= MOESQ_PERMUTE_NOALLOC_MAX_COUNTS, else
 *   MOESQ_ERR_CAPACITY is returned and nothing is enqueued (e.g. E = 512 allows
 *   T*k up to 524288).
 *   The first call on a device looks up the array's device address with that device
 *   current (cudaGetSymbolAddress) and caches it for the process; make that first call
 *   before any stream capture.  The cached address belongs to the device's primary
 *   context: calls after cudaDeviceReset in the same process are not supported.
 *   Every GPU that loads the library holds the array until the process exits.  All
 *   calls share it, and each call overwrites the parts it reads,
 *   so calls whose executions overlap on the GPU (other streams, other host threads)
 *   race and must be ordered by the caller. */
#define MOESQ_PERMUTE_NOALLOC_MAX_COUNTS 262144
moesq_status moesq_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                   int32_t* expert_offsets, int32_t* pad_offsets,
                                   int32_t* slot_token, int32_t* token_slot, int32_t* d_status,
                                   moesq_stream_t stream);

/* Upper bound of the padded row count for S slots over E experts. */
int64_t moesq_padded_rows(int64_t S, int32_t E);

/* Weighted combine: out[t] = bf16( sum_j w[t,j] * y[token_slot[t,j]] ), float32, j order.
 *   y device bf16 [S, H];  token_slot device i32 [T, k];  topk_w device f32 [T, k];
 *   out device bf16 [T, H].  H % 8 == 0. */
moesq_status moesq_unpermute(const uint16_t* y, const int32_t* token_slot, const float* topk_w,
                             int64_t T, int32_t k, int64_t H, uint16_t* out,
                             moesq_stream_t stream);

/* ------------------------------------------------------------------------- *
 * Activation quantisation  [format] ("dynamic per-32 group scales, FP32
 * per-tensor global scale stored per expert linear")
 * ------------------------------------------------------------------------- */

typedef enum moesq_sf_layout {
  MOESQ_SF_LINEAR = 0, /* codes [rows, K/2], scales [rows, K/32], row = output row index */
  MOESQ_SF_KERNEL = 1  /* padded GEMM operand: codes [P, K/2] at row p = pad_offsets[e] +
                          (s - expert_offsets[e]); scales in 512-byte blocks
                          [P/128][K/128][512], row r scale j at (r%32)*16+(r/32)*4+j */
} moesq_sf_layout;

/* bf16 -> NVFP4 codes + E4M3 per-32 scales, one output row per slot.
 *   x              device bf16 [T, K]
 *   gather         device i32 [rows] (row of x for each output row) or NULL (identity)
 *   expert_offsets device i32 [E+1] or NULL (then every row uses g_in[0])
 *   pad_offsets    device i32 [E+1], required for MOESQ_SF_KERNEL
 *   g_in           device f32 [E] (or [1] without expert_offsets): input globals
 *   codes, sf      device outputs in the chosen layout
 * K % 128 == 0. */
moesq_status moesq_quant_act(const uint16_t* x, int64_t K, const int32_t* gather,
                             const int32_t* expert_offsets, const int32_t* pad_offsets,
                             int32_t E, const float* g_in, int64_t rows, int32_t layout,
                             uint8_t* codes, uint8_t* sf, moesq_stream_t stream);

/* Token-major variant used by moesq_moe_forward: reads each token row of x once and
 * writes one padded operand row per routed slot (MOESQ_SF_KERNEL layout only).
 *   x          device bf16 [T, K];  topk_ids, token_slot  device i32 [T, k]
 *   expert_offsets, pad_offsets  device i32 [E+1] (moesq_permute);  g_in device f32 [E]
 *   codes, sf  padded operand outputs as for MOESQ_SF_KERNEL.
 * Same arithmetic as moesq_quant_act; ids outside [0, E) are treated as expert 0.
 * One kernel launch, or two when K % 1024 == 0, k <= 32 and the codes written reach 64
 * MiB (the scales are then written as rows and rearranged into the tensor-core blocks
 * in place by a second kernel on the same stream); sf's padding rows hold no values. */
moesq_status moesq_quant_act_routed(const uint16_t* x, int64_t T, int64_t K,
                                    const int32_t* topk_ids, const int32_t* token_slot, int32_t k,
                                    const int32_t* expert_offsets, const int32_t* pad_offsets,
                                    int32_t E, const float* g_in, uint8_t* codes, uint8_t* sf,
                                    moesq_stream_t stream);

/* ------------------------------------------------------------------------- *
 * Grouped sparse GEMM  [kernel]
 * ------------------------------------------------------------------------- */

typedef struct moesq_linear {
  const uint8_t* packed; /* device u8 [E, out, K/4]  weight_sparse_packed, used as stored */
  const uint8_t* meta;   /* device, moesq_repack_meta output */
  const uint8_t* sf;     /* device, moesq_repack_meta output */
  const float* alpha_w;  /* device f32 [E]; [E, 2] (gate, up) for GATE_UP_EXACT */
  int64_t out;           /* output features (2I for gate_up) */
  int64_t K;             /* dense K */
  int32_t E;             /* experts */
  int32_t kind;          /* moesq_linear_kind (GATE_UP_SPLIT behaves as GATE_UP here; GATE_UP_EXACT
                            scales the up half by its own global) */
} moesq_linear;

typedef enum moesq_epilogue {
  MOESQ_EPI_F32 = 0,         /* out f32 [S, W.out], row = slot, column = original weight row */
  MOESQ_EPI_BF16 = 1,        /* out bf16 [S, W.out] */
  MOESQ_EPI_SWIGLU_NVFP4 = 2 /* gate_up only: h = silu(gate)*up requantised with g_next[e]:
                                out u8 codes [P, I/2] (padded rows), out_sf blocks
                                [P/128][I/128][512] -- the next GEMM's B operand.
                                h is fp32 (exponential and reciprocal of the SiLU on
                                the MUFU, a few ulp); the NVFP4 rule runs on h with
                                the accumulator scales folded into its amax and code
                                multiplier, so it matches the rule on the exact h
                                except where h lies within that error of a rounding
                                boundary */
} moesq_epilogue;

/* y[s, m] = g_act[e] * alpha_w[e] * sum_k W_e[m, k] * A[s, k] for every slot s of expert e.
 *   act_codes  device u8 [P_cap, K/2] padded rows (moesq_quant_act, MOESQ_SF_KERNEL)
 *   act_sf     device u8 [P_cap/128][K/128][512]
 *   g_act      device f32 [E]
 *   expert_offsets, pad_offsets  device i32 [E+1] (moesq_permute)
 *   S          number of slots (expert_offsets[E]); P_cap = padded row capacity of the
 *              act/out buffers, >= moesq_padded_rows(S, E) and a multiple of 128
 *   g_next     device f32 [E] (SWIGLU only, else NULL)
 *   ws         device workspace of moesq_grouped_gemm_workspace_size() bytes (may be 0)
 * Weights are the sparse operand A of tcgen05.mma.sp (M = weight rows), tokens are
 * B (N).  out % 128 == 0, K % 128 == 0, out % 256 == 0 for SWIGLU.
 * Bounded waits that give up raise MOESQ_DFLAG_TIMEOUT. */
moesq_status moesq_grouped_gemm(const moesq_linear* W, const uint8_t* act_codes,
                                const uint8_t* act_sf, const float* g_act,
                                const int32_t* expert_offsets, const int32_t* pad_offsets,
                                int64_t S, int64_t P_cap, int32_t epilogue, const float* g_next,
                                void* out, uint8_t* out_sf, void* ws, size_t ws_bytes,
                                int32_t* d_status, moesq_stream_t stream);
moesq_status moesq_grouped_gemm_workspace_size(const moesq_linear* W, int64_t S, size_t* bytes);

/* Launch shape of the grouped GEMMs (the pages have no counterpart; these calls
 * exist so that tests can make every CTA pair run several work items).  A
 * grouped GEMM launches one persistent CTA pair per two SMs that the device
 * holds at once, and each pair walks the (expert, token tile, weight-tile pair)
 * work items pid, pid + npairs, ...
 *   moesq_set_gemm_pair_limit: caps npairs for every later launch in the process
 *     (0 = no cap, the default).  The result of a GEMM does not depend on npairs.
 *     Launches already queued keep the npairs they were launched with;
 *     max_pairs >= 0.
 *   moesq_gemm_launch_pairs: npairs that a launch on the current device would use
 *     now (cap applied), for the sparse (dense = 0) or the dense comparison kernel
 *     with the given epilogue. */
moesq_status moesq_set_gemm_pair_limit(int32_t max_pairs);
moesq_status moesq_gemm_launch_pairs(int32_t dense, int32_t epilogue, int32_t* pairs);

/* Down GEMM with the weighted combine fused into its epilogue (the combine of the
 * MoESQ README "Kernels" path, done where y is produced): out[t, :] = sum over j in
 * 0..k-1, in that order, of topk_w[t, j] * y[token_slot[t, j], :], float32 products of
 * the stored bf16 y without fused multiply-add, rounded once to bf16 -- bit-identical
 * to moesq_grouped_gemm(MOESQ_EPI_BF16) followed by moesq_unpermute.  Deterministic:
 * every (token, 128-output tile) counts its k slot arrivals (each after that slot's y
 * row is written and fenced) and the arrival that completes the count sums the k rows.
 *   W          MOESQ_LINEAR_DOWN weights; other GEMM arguments as moesq_grouped_gemm
 *   S          == T * k, 1 <= k <= 32
 *   slot_token, token_slot   moesq_permute's outputs for this batch (device i32)
 *   topk_w     device f32 [T, k]
 *   y          device bf16 [S, W.out] scratch: every slot's row, as MOESQ_EPI_BF16 writes it
 *   out        device bf16 [T, W.out]
 *   arrivals   device i32 [T * W.out / 128] scratch, zeroed by this call (stream-ordered)
 * Returns as moesq_grouped_gemm; the fused epilogue writes y rows straight from
 * registers (no staging), so on large batches it runs slower than the two kernels
 * (the library's forward keeps them separate). */
moesq_status moesq_grouped_gemm_down_combine(const moesq_linear* W, const uint8_t* act_codes,
                                             const uint8_t* act_sf, const float* g_act,
                                             const int32_t* expert_offsets, const int32_t* pad_offsets,
                                             int64_t S, int64_t P_cap, const int32_t* slot_token,
                                             const int32_t* token_slot, const float* topk_w, int64_t T,
                                             int32_t k, uint16_t* y, uint16_t* out, int32_t* arrivals,
                                             int32_t* d_status, moesq_stream_t stream);

/* Measured rate of the sparse block-scaled FP4 tensor-core MMA (the roofline
 * denominator of the grouped GEMMs, with 8 x the measured bf16 GEMM rate as a floor):
 * every CTA pair of the device issues `iters` x 4 tcgen05.mma.sp (cta_group::2,
 * kind::mxf4nvf4, M = 256, dense K = 128, N = n) back to back on operands already in
 * shared memory and TMEM, after one untimed launch.  Writes dense-equivalent TFLOP/s
 * (2 M N K per MMA) to *tflops.  Synchronises the stream (a measurement call, not part
 * of the hot path); a bounded wait that gives up raises MOESQ_DFLAG_TIMEOUT in d_status
 * (may be NULL).  iters >= 1, 16 <= n <= 256, n % 16 == 0. */
moesq_status moesq_measure_sparse_mma_peak(int32_t iters, int32_t n, double* tflops, int32_t* d_status,
                                           moesq_stream_t stream);

/* Work-item width of the sparse SwiGLU gate_up GEMM (the pages have no counterpart).
 * A work item is one weight-tile pair times one 128-token tile, or, on large batches,
 * two 128-token tiles of one expert computed by single MMAs of N <= 256 ("wide" items:
 * the weight tile is read from shared memory once per 256 tokens).  Wide items need
 * K % 512 == 0; without a forced width they are chosen when K >= 4096 and
 * S >= 256 * E.  The result
 * of a GEMM does not depend on the width.
 *   moesq_set_gemm_tiles_per_item: 0 = choose (the default), 1 = one tile, 2 = wide
 *     wherever the shape allows, for every later launch in the process; tiles in 0..2.
 *   moesq_gemm_tiles_per_item: the width (1 or 2) that a launch with these arguments
 *     would use now (dense != 0: the dense comparison kernel, always 1). */
moesq_status moesq_set_gemm_tiles_per_item(int32_t tiles);
moesq_status moesq_gemm_tiles_per_item(int32_t dense, int32_t epilogue, int64_t K, int64_t E, int64_t S,
                                       int32_t* tiles);

/* Dense comparison GEMM: the same grouped GEMM, epilogues and argument meanings on
 * dense NVFP4 weights, the pages' alternative storage ("--no-sparse-storage writes
 * dense packed NVFP4 with the pruned elements zeroed", Usage of the MoESQ repository
 * README), with the dense tensor-core MMA (kind::mxf4nvf4, 64 dense K per MMA).
 *   W->packed  device u8 [E, out, K/2] dense codes (moesq_decode of the sparse storage),
 *              same tile row order as the sparse operand; W->meta is not used
 *   W->sf, act_sf  scale blocks of 16 elements (moesq_sf_expand_block16 of the 32-element
 *              blocks: [rows/128][K/64][512])
 * The result equals the sparse GEMM's (same decoded weights and scales) up to the
 * FP32 accumulation order.  Returns as moesq_grouped_gemm. */
moesq_status moesq_grouped_gemm_dense(const moesq_linear* W, const uint8_t* act_codes,
                                      const uint8_t* act_sf, const float* g_act,
                                      const int32_t* expert_offsets, const int32_t* pad_offsets,
                                      int64_t S, int64_t P_cap, int32_t epilogue, const float* g_next,
                                      void* out, uint8_t* out_sf, int32_t* d_status,
                                      moesq_stream_t stream);

/* Routed NVFP4 rows quantised elsewhere (e.g. received from the GPU that holds the
 * tokens) -> the padded operand layout of moesq_grouped_gemm.
 *   codes_in device u8 [n, K/2], sf_in device u8 [n, K/32] (linear, MOESQ_SF_LINEAR)
 *   gather   device i32 [S]: input row of slot s, slots in expert order (moesq_permute's
 *            slot_token of the received rows)
 *   expert_offsets, pad_offsets device i32 [E+1] (moesq_permute)
 *   codes_out device u8 [P, K/2], sf_out device u8 [P/128][K/128][512] (MOESQ_SF_KERNEL)
 * K % 128 == 0; codes 16-byte aligned.  Bytes are copied unchanged. */
moesq_status moesq_gather_act(const uint8_t* codes_in, const uint8_t* sf_in, const int32_t* gather,
                              int64_t S, int64_t K, const int32_t* expert_offsets,
                              const int32_t* pad_offsets, int32_t E, uint8_t* codes_out, uint8_t* sf_out,
                              moesq_stream_t stream);

/* 32-element scale blocks -> 16-element scale blocks for the dense MMA: each 512-byte
 * block b (128 rows x 4 scales, one per 32 K: row r, scale j at (r%32)*16 + (r/32)*4 + j)
 * becomes blocks 2b and 2b+1 (one scale per 16 K, each 32-element scale written twice).
 *   sf32 device u8 [nblocks * 512];  sf16 device u8 [2 * nblocks * 512]; 16-byte aligned. */
moesq_status moesq_sf_expand_block16(const uint8_t* sf32, uint8_t* sf16, int64_t nblocks,
                                     moesq_stream_t stream);

/* ------------------------------------------------------------------------- *
 * The whole routed-expert MLP of one MoE layer
 * ------------------------------------------------------------------------- */

typedef struct moesq_moe_layer {
  int32_t E, k;
  int64_t H, I;
  moesq_linear gate_up;      /* out = 2I, K = H, kind GATE_UP or GATE_UP_SPLIT (already folded) */
  moesq_linear down;         /* out = H, K = I */
  const float* g_in_gate_up; /* device f32 [E] static input globals of gate_up */
  const float* g_in_down;    /* device f32 [E] static input globals of down */
} moesq_moe_layer;

/* permute -> quant_act -> gate_up (fused SwiGLU + NVFP4 requant) -> down -> combine.
 *   x device bf16 [T, H];  topk_ids device i32 [T, k];  topk_w device f32 [T, k]
 *   out device bf16 [T, H];  ws device workspace of moesq_moe_forward_workspace_size(). */
moesq_status moesq_moe_forward(const moesq_moe_layer* L, const uint16_t* x,
                               const int32_t* topk_ids, const float* topk_w, int64_t T,
                               uint16_t* out, void* ws, size_t ws_bytes, int32_t* d_status,
                               moesq_stream_t stream);
moesq_status moesq_moe_forward_workspace_size(const moesq_moe_layer* L, int64_t T,
                                              size_t* bytes);

/* Same as moesq_moe_forward with HOST inputs and output.  The batch is cut into
 * token chunks (at least 2048 tokens, at most 8 chunks); for each, x/topk_ids/topk_w
 * are copied host->device into `ws`, the layer runs on `stream`, and out is copied
 * back to the host buffer.  The uploads and downloads run on two internal streams of
 * the current device (created on the first call and kept for the process), ordered
 * against `stream` by events, so the copies of one chunk overlap the forward of
 * another.  The copies start after the work already queued on `stream`; the call
 * returns after everything it queued has completed (it synchronises all three
 * streams, also on error).  The output equals moesq_moe_forward's bit for bit: a
 * token's result depends only on its own row and routing.  `ws` holds the forward
 * workspace of one chunk and one input/output buffer set per chunk, so no upload
 * waits for an earlier chunk's download (see moesq_moe_forward_host_workspace_size).  Host buffers should be pinned: pageable
 * ones are copied correctly but without overlap. */
moesq_status moesq_moe_forward_host(const moesq_moe_layer* L, const uint16_t* h_x,
                                    const int32_t* h_topk_ids, const float* h_topk_w,
                                    int64_t T, uint16_t* h_out, void* ws, size_t ws_bytes,
                                    int32_t* d_status, moesq_stream_t stream);
moesq_status moesq_moe_forward_host_workspace_size(const moesq_moe_layer* L, int64_t T,
                                                   size_t* bytes);

/* ------------------------------------------------------------------------- *
 * Self-test of the failure path
 * ------------------------------------------------------------------------- */

/* Runs the library's three bounded mbarrier waits (the ones every pipeline wait goes
 * through) on a barrier phase that nothing completes.  Each gives up after limit_ns
 * (0 < limit_ns <= 1e8; polling checks the clock every few tries, so the kernel runs
 * a small multiple of limit_ns), ORs MOESQ_DFLAG_TIMEOUT into *d_status and writes 1
 * to d_gave_up[i] (device i32 [3]: suspending, spinning, polling wait).  The kernel
 * returns normally: no fault, no trap. */
moesq_status moesq_selftest_wait_timeout(int32_t* d_status, int64_t limit_ns, int32_t* d_gave_up,
                                         moesq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOESQ_H */
