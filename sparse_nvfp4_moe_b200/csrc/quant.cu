// Dynamic NVFP4 activation quantisation (bf16 -> E2M1 codes + E4M3 per-32 scales).
//
// "Activations: NVFP4, dynamic per-32 group scales, FP32 per-tensor global scale
// stored per expert linear" ("Compression details" table, Qwen3.5-397B-A17B-
// P48NVFP4-MoESQ model card).  One output row per routed slot: the row of x of
// its token is gathered and quantised with the input global of its expert.  One
// thread per 32-element group: 64 bytes of bf16 in (4 x 16-byte loads, a warp
// reads 2 KB contiguous), 16 bytes of codes and one scale byte out.  In the
// KERNEL layout rows land in the padded, 128-row aligned GEMM operand buffer
// and scales in the 512-byte tensor-core scale-factor blocks.
#include "common.cuh"

namespace moesq {

__device__ __forceinline__ int find_expert(const int32_t* __restrict__ off, int E, int64_t s) {
  int lo = 0, hi = E - 1;  // largest e with off[e] <= s
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= s) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void k_quant_act(const uint16_t* __restrict__ x, int64_t K, const int32_t* __restrict__ gather,
                            const int32_t* __restrict__ expert_offsets,
                            const int32_t* __restrict__ pad_offsets, int E,
                            const float* __restrict__ g_in, int64_t rows, int layout,
                            uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  const int64_t G = K / 32;
  const int64_t n = rows * G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t s = i / G, grp = i % G;
    const int64_t src = gather ? (int64_t)gather[s] : s;
    int e = 0;
    if (expert_offsets) e = find_expert(expert_offsets, E, s);
    const float g = g_in[e];
    float v[32];
    const uint4* q = reinterpret_cast<const uint4*>(x + src * K + 32 * grp);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = q[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * c + 2 * j] = bf16_bits_to_float(w[j] & 0xFFFF);
        v[8 * c + 2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const GroupScale gs = nvfp4_group_scale(amax, g);
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) o[c] = nvfp4_word(v + 8 * c, gs.inv);
    int64_t row = s;
    if (layout == MOESQ_SF_KERNEL) row = (int64_t)pad_offsets[e] + (s - expert_offsets[e]);
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + 16 * grp) = make_uint4(o[0], o[1], o[2], o[3]);
    if (layout == MOESQ_SF_KERNEL) {
      const int64_t blk = (row / 128) * (K / 128) + grp / 4;
      sf[blk * 512 + sf_block_offset((uint32_t)(row % 128), (uint32_t)(grp % 4))] = (uint8_t)gs.sc;
    } else {
      sf[s * G + grp] = (uint8_t)gs.sc;
    }
  }
}

// Token-major variant for the MoE forward: thread per (token, 32-group); x is
// read once per token and written once per routed slot (k times), each with the
// global of the slot's expert, into the padded operand layout.
template <bool BATCHED>
__global__ void k_quant_act_routed(const uint16_t* __restrict__ x, int64_t T, int64_t K,
                                   const int32_t* __restrict__ topk_ids,
                                   const int32_t* __restrict__ token_slot, int k,
                                   const int32_t* __restrict__ expert_offsets,
                                   const int32_t* __restrict__ pad_offsets, int E,
                                   const float* __restrict__ g_in, uint8_t* __restrict__ codes,
                                   uint8_t* __restrict__ sf) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  const int64_t G = K / 32;
  const int64_t n = T * G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / G, grp = i % G;
    float v[32];
    const uint4* q = reinterpret_cast<const uint4*>(x + t * K + 32 * grp);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = q[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * c + 2 * j] = bf16_bits_to_float(w[j] & 0xFFFF);
        v[8 * c + 2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    // the codes and scale depend on the slot only through its expert's global: a
    // slot whose global equals the previous slot's (bit for bit) reuses them
    float g_prev = 0.0f;
    GroupScale gs = {0u, 0.0f};
    uint32_t o[4] = {0u, 0u, 0u, 0u};
    if constexpr (!BATCHED) {
      // large batches: one slot at a time (fewer registers, more warps to hide latency)
      for (int j = 0; j < k; ++j) {
        int e = topk_ids[t * k + j];
        if (e < 0 || e >= E) e = 0;
        const int64_t s = token_slot[t * k + j];
        const float g = g_in[e];
        if (j == 0 || __float_as_uint(g) != __float_as_uint(g_prev)) {
          g_prev = g;
          gs = nvfp4_group_scale(amax, g);
#pragma unroll
          for (int c = 0; c < 4; ++c) o[c] = nvfp4_word(v + 8 * c, gs.inv);
        }
        const int64_t row = (int64_t)pad_offsets[e] + (s - expert_offsets[e]);
        *reinterpret_cast<uint4*>(codes + row * (K / 2) + 16 * grp) = make_uint4(o[0], o[1], o[2], o[3]);
        const int64_t blk = (row / 128) * (K / 128) + grp / 4;
        sf[blk * 512 + sf_block_offset((uint32_t)(row % 128), (uint32_t)(grp % 4))] = (uint8_t)gs.sc;
      }
    } else {
      // slots in chunks of 8: all index and table loads of a chunk are issued before any
      // is used, so a small batch waits for two load round trips per chunk, not per slot
      for (int j0 = 0; j0 < k; j0 += 8) {
        int ev[8];
        int64_t rowv[8];
        float gv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          int e = j < k ? topk_ids[t * k + j] : 0;
          ev[u] = (e < 0 || e >= E) ? 0 : e;
          rowv[u] = j < k ? (int64_t)token_slot[t * k + j] : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          gv[u] = g_in[ev[u]];
          rowv[u] += (int64_t)pad_offsets[ev[u]] - expert_offsets[ev[u]];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          if (j < k) {
            const float g = gv[u];
            if (j == 0 || __float_as_uint(g) != __float_as_uint(g_prev)) {
              g_prev = g;
              gs = nvfp4_group_scale(amax, g);
#pragma unroll
              for (int c = 0; c < 4; ++c) o[c] = nvfp4_word(v + 8 * c, gs.inv);
            }
            const int64_t row = rowv[u];
            *reinterpret_cast<uint4*>(codes + row * (K / 2) + 16 * grp) = make_uint4(o[0], o[1], o[2], o[3]);
            const int64_t blk = (row / 128) * (K / 128) + grp / 4;
            sf[blk * 512 + sf_block_offset((uint32_t)(row % 128), (uint32_t)(grp % 4))] = (uint8_t)gs.sc;
          }
        }
      }
    }
  }
}

// Warp form of the routed quantisation for K % 1024 == 0 (a warp covers 32 groups =
// 1024 elements of one token).  Lanes 0..k-1 load the token's routing once (expert,
// slot, the expert's global and padded row) and the warp shares it by shuffles, so a
// thread waits for one round of index loads per token instead of two per slot.  Each
// lane quantises its group and stores 16 code bytes per slot (512 contiguous bytes per
// warp and slot); lanes 4m..4m+3 hold the four scales that share a 512-byte block
// position and lane 4m stores them as one 32-bit word.
//
// On large batches (`rows`) the scales go out as rows first: lane 4m's word lands at
// bytes 32c + 4m of its slot's padded row of K/32 scale bytes (one 32-byte sector per
// warp and slot), and k_sf_rows_to_blocks then rearranges each 128-row slab, in place,
// into the 512-byte tensor-core blocks.  Written straight into the blocks, a slot's 32
// words land in 32 different 32-byte sectors, each completed by 8 slots of other tokens
// written at other times; once the codes streaming through L2 evict the partly written
// sectors before they are complete, the scale stores, 4% of the bytes, took 44% of the
// kernel's time (Qwen3-235B-A22B T = 65536: 483 us with them, 270 us without).  Small
// batches, whose scales stay in L2, write the blocks directly and save the second kernel.
__global__ void k_quant_act_routed_warp(const uint16_t* __restrict__ x, int64_t T, int64_t K,
                                        const int32_t* __restrict__ topk_ids,
                                        const int32_t* __restrict__ token_slot, int k,
                                        const int32_t* __restrict__ expert_offsets,
                                        const int32_t* __restrict__ pad_offsets, int E,
                                        const float* __restrict__ g_in, uint8_t* __restrict__ codes,
                                        uint8_t* __restrict__ sf, bool rows) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t W = K / 1024;  // warp chunks per token
  const int64_t nw = T * W;
  const int64_t wstride = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < nw; w += wstride) {
    const int64_t t = w / W;
    const int64_t grp = 32 * (w - t * W) + lane;
    // routing of token t: lane j < k holds slot j's global and padded row
    float gj = 0.0f;
    int rowj = 0;
    if (lane < k) {
      int e = topk_ids[t * k + lane];
      if (e < 0 || e >= E) e = 0;
      gj = g_in[e];
      rowj = pad_offsets[e] + (token_slot[t * k + lane] - expert_offsets[e]);
    }
    float v[32];
    const uint4* q = reinterpret_cast<const uint4*>(x + t * K + 32 * grp);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = q[c];
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * c + 2 * j] = bf16_bits_to_float(wd[j] & 0xFFFF);
        v[8 * c + 2 * j + 1] = bf16_bits_to_float(wd[j] >> 16);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    // the codes and scale depend on the slot only through its expert's global: a slot
    // whose global equals the previous slot's (bit for bit) reuses them (warp-uniform)
    float g_prev = 0.0f;
    GroupScale gs = {0u, 0.0f};
    uint32_t o[4] = {0u, 0u, 0u, 0u};
    uint32_t word = 0u;
    for (int j = 0; j < k; ++j) {
      const float g = __shfl_sync(0xffffffffu, gj, j);
      const int64_t row = __shfl_sync(0xffffffffu, rowj, j);
      if (j == 0 || __float_as_uint(g) != __float_as_uint(g_prev)) {
        g_prev = g;
        gs = nvfp4_group_scale(amax, g);
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = nvfp4_word(v + 8 * c, gs.inv);
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, gs.sc, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, gs.sc, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, gs.sc, 3);
        word = (gs.sc & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
      }
      *reinterpret_cast<uint4*>(codes + row * (K / 2) + 16 * grp) = make_uint4(o[0], o[1], o[2], o[3]);
      if ((lane & 3) == 0) {
        if (rows) {
          *reinterpret_cast<uint32_t*>(sf + row * (K / 32) + grp) = word;
        } else {
          const int64_t blk = (row / 128) * (K / 128) + grp / 4;
          *reinterpret_cast<uint32_t*>(sf + blk * 512 + sf_block_offset((uint32_t)(row % 128), 0u)) = word;
        }
      }
    }
  }
}

// In place, per 128-row slab of the scale buffer: rows of K/32 scale bytes (row r of the
// slab at r * K/32) into the slab's K/128 blocks of 512 bytes (row r, scale j of block kk
// at kk * 512 + (r % 32) * 16 + (r / 32) * 4 + j).  Both layouts of a slab fill the same
// 128 * K/32 bytes at the same offset.  One block of threads per slab: coalesced 16-byte
// loads into shared memory (rows padded by 4 bytes so that the gather is conflict-free),
// then each thread writes one 16-byte piece (rows r, r + 32, r + 64, r + 96 of one block).
// The slab count comes from pad_offsets[E] on the device.
__global__ void k_sf_rows_to_blocks(uint8_t* __restrict__ sf, const int32_t* __restrict__ pad_offsets, int E,
                                    int64_t K) {
  extern __shared__ __align__(16) uint8_t rows[];
  pdl_wait();
  pdl_trigger();
  const int rb = (int)(K / 32);   // bytes per row
  const int rs = rb + 4;          // padded row stride in shared memory
  const int64_t slab_bytes = (int64_t)128 * rb;
  const int64_t nslab = pad_offsets[E] / 128;
  for (int64_t b = blockIdx.x; b < nslab; b += gridDim.x) {
    uint8_t* g = sf + b * slab_bytes;
    for (int i = threadIdx.x; i < 128 * rb / 16; i += blockDim.x) {
      const int r = (16 * i) / rb, c = (16 * i) % rb;
      const uint4 v = *reinterpret_cast<const uint4*>(g + 16 * (int64_t)i);
      uint32_t* d = reinterpret_cast<uint32_t*>(rows + r * rs + c);  // rs is 4-byte aligned only
      d[0] = v.x;
      d[1] = v.y;
      d[2] = v.z;
      d[3] = v.w;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 128 * rb / 16; i += blockDim.x) {
      const int kk = i / 32, r = i % 32;  // block kk, rows r + 32m: 16 bytes at kk * 512 + 16 r
      uint4 v;
      v.x = *reinterpret_cast<const uint32_t*>(rows + r * rs + 4 * kk);
      v.y = *reinterpret_cast<const uint32_t*>(rows + (r + 32) * rs + 4 * kk);
      v.z = *reinterpret_cast<const uint32_t*>(rows + (r + 64) * rs + 4 * kk);
      v.w = *reinterpret_cast<const uint32_t*>(rows + (r + 96) * rs + 4 * kk);
      *reinterpret_cast<uint4*>(g + (int64_t)kk * 512 + 16 * r) = v;
    }
    __syncthreads();
  }
}

// Routed NVFP4 rows quantised elsewhere (codes [n, K/2], linear scales [n, K/32], e.g.
// received from another GPU) into the grouped GEMM's padded operand layout: slot s of
// the expert-ordered list takes input row gather[s] and lands on padded row
// pad_offsets[e] + (s - expert_offsets[e]).  Thread per (slot, 32-element group): one
// 16-byte code chunk and one scale byte.
__global__ void k_gather_act(const uint8_t* __restrict__ codes_in, const uint8_t* __restrict__ sf_in,
                             const int32_t* __restrict__ gather, int64_t S, int64_t K,
                             const int32_t* __restrict__ expert_offsets, const int32_t* __restrict__ pad_offsets,
                             int E, uint8_t* __restrict__ codes_out, uint8_t* __restrict__ sf_out) {
  pdl_wait();
  pdl_trigger();
  const int64_t G = K / 32;
  const int64_t n = S * G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t s = i / G, grp = i % G;
    const int64_t src = gather[s];
    const int e = find_expert(expert_offsets, E, s);
    const int64_t row = (int64_t)pad_offsets[e] + (s - expert_offsets[e]);
    *reinterpret_cast<uint4*>(codes_out + row * (K / 2) + 16 * grp) =
        *reinterpret_cast<const uint4*>(codes_in + src * (K / 2) + 16 * grp);
    const int64_t blk = (row / 128) * (K / 128) + grp / 4;
    sf_out[blk * 512 + sf_block_offset((uint32_t)(row % 128), (uint32_t)(grp % 4))] = sf_in[src * G + grp];
  }
}

// 32-element scale blocks -> 16-element scale blocks: thread per (block, lane l),
// one 16-byte row of four 4-scale words in, one such row out to each of the two
// blocks (scales 0,0,1,1 and 2,2,3,3 of every word)
__global__ void k_sf_expand_block16(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = in[i];
    const int64_t b = i >> 5, l = i & 31;
    out[(2 * b) * 32 + l] = make_uint4(__byte_perm(v.x, 0, 0x1100), __byte_perm(v.y, 0, 0x1100),
                                       __byte_perm(v.z, 0, 0x1100), __byte_perm(v.w, 0, 0x1100));
    out[(2 * b + 1) * 32 + l] = make_uint4(__byte_perm(v.x, 0, 0x3322), __byte_perm(v.y, 0, 0x3322),
                                           __byte_perm(v.z, 0, 0x3322), __byte_perm(v.w, 0, 0x3322));
  }
}

}  // namespace moesq

using namespace moesq;

extern "C" moesq_status moesq_gather_act(const uint8_t* codes_in, const uint8_t* sf_in, const int32_t* gather,
                                         int64_t S, int64_t K, const int32_t* expert_offsets,
                                         const int32_t* pad_offsets, int32_t E, uint8_t* codes_out,
                                         uint8_t* sf_out, moesq_stream_t stream) {
  MOESQ_REQUIRE(S >= 0 && K >= 0 && E >= 1, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 128 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (S == 0 || K == 0) return MOESQ_OK;
  MOESQ_REQUIRE(codes_in && sf_in && gather && expert_offsets && pad_offsets && codes_out && sf_out,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(codes_in) && moesq_aligned16(codes_out) && moesq_aligned16(sf_out),
                MOESQ_ERR_INVALID_ARG);
  const int64_t n = S * (K / 32);
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  if (moesq_launch(k_gather_act, dim3((unsigned)g), dim3(256), 0, (cudaStream_t)stream, codes_in, sf_in, gather, S, K,
                   expert_offsets, pad_offsets, (int)E, codes_out, sf_out) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_sf_expand_block16(const uint8_t* sf32, uint8_t* sf16, int64_t nblocks,
                                                moesq_stream_t stream) {
  MOESQ_REQUIRE(nblocks >= 0, MOESQ_ERR_INVALID_ARG);
  if (nblocks == 0) return MOESQ_OK;
  MOESQ_REQUIRE(sf32 && sf16 && moesq_aligned16(sf32) && moesq_aligned16(sf16), MOESQ_ERR_INVALID_ARG);
  const int64_t n = nblocks * 32;
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  if (moesq_launch(k_sf_expand_block16, dim3((unsigned)g), dim3(256), 0, (cudaStream_t)stream,
                   reinterpret_cast<const uint4*>(sf32), reinterpret_cast<uint4*>(sf16), n) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_quant_act_routed(const uint16_t* x, int64_t T, int64_t K,
                                               const int32_t* topk_ids, const int32_t* token_slot,
                                               int32_t k, const int32_t* expert_offsets,
                                               const int32_t* pad_offsets, int32_t E,
                                               const float* g_in, uint8_t* codes, uint8_t* sf,
                                               moesq_stream_t stream) {
  MOESQ_REQUIRE(T >= 0 && K >= 0 && k >= 1 && E >= 1, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 128 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (T == 0 || K == 0) return MOESQ_OK;
  MOESQ_REQUIRE(x && topk_ids && token_slot && expert_offsets && pad_offsets && g_in && codes && sf,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(x) && moesq_aligned16(codes) && moesq_aligned16(sf),
                MOESQ_ERR_INVALID_ARG);
  const int64_t n = T * (K / 32);
  int64_t g = (n + 127) / 128;
  if (g > 148 * 32) g = 148 * 32;
  // a warp per 1024 elements of a token when K allows it and k fits a warp; otherwise
  // thread per group: for small batches (decode) every slot's index loads in flight at
  // once, for large ones more warps
  if (K % 1024 == 0 && k <= 32) {
    // scales as rows first once the codes written (S K/2 bytes) are half of L2 or more
    const bool rows = T * k * (K / 2) >= ((int64_t)64 << 20);
    if (moesq_launch(k_quant_act_routed_warp, dim3((unsigned)g), dim3(128), 0, (cudaStream_t)stream, x, T, K, topk_ids,
                     token_slot, k, expert_offsets, pad_offsets, E, g_in, codes, sf, rows) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    if (!rows) return MOESQ_OK;
    // the slabs: at most ceil((T k + 127 E) / 128) of them; a block per slab, up to 8 a SM
    const size_t smem = (size_t)128 * (K / 32 + 4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_sf_rows_to_blocks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    int64_t slabs = (T * k + 127 * (int64_t)E) / 128 + 1;
    if (slabs > 148 * 8) slabs = 148 * 8;
    if (moesq_launch(k_sf_rows_to_blocks, dim3((unsigned)slabs), dim3(256), smem, (cudaStream_t)stream, sf, pad_offsets,
                     E, K) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    return MOESQ_OK;
  }
  const cudaError_t err =
      T <= 512 ? moesq_launch(k_quant_act_routed<true>, dim3((unsigned)g), dim3(128), 0, (cudaStream_t)stream, x, T, K,
                              topk_ids, token_slot, k, expert_offsets, pad_offsets, E, g_in, codes, sf)
               : moesq_launch(k_quant_act_routed<false>, dim3((unsigned)g), dim3(128), 0, (cudaStream_t)stream, x, T, K,
                              topk_ids, token_slot, k, expert_offsets, pad_offsets, E, g_in, codes, sf);
  if (err != cudaSuccess) return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_quant_act(const uint16_t* x, int64_t K, const int32_t* gather,
                                        const int32_t* expert_offsets, const int32_t* pad_offsets,
                                        int32_t E, const float* g_in, int64_t rows, int32_t layout,
                                        uint8_t* codes, uint8_t* sf, moesq_stream_t stream) {
  MOESQ_REQUIRE(K >= 0 && rows >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(layout == MOESQ_SF_LINEAR || layout == MOESQ_SF_KERNEL, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 128 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (rows == 0 || K == 0) return MOESQ_OK;
  MOESQ_REQUIRE(x && g_in && codes && sf, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(x) && moesq_aligned16(codes) && moesq_aligned16(sf),
                MOESQ_ERR_INVALID_ARG);
  if (expert_offsets) MOESQ_REQUIRE(E >= 1, MOESQ_ERR_INVALID_ARG);
  if (layout == MOESQ_SF_KERNEL) MOESQ_REQUIRE(expert_offsets && pad_offsets, MOESQ_ERR_INVALID_ARG);
  const int64_t n = rows * (K / 32);
  int64_t g = (n + 127) / 128;
  if (g > 148 * 32) g = 148 * 32;
  if (moesq_launch(k_quant_act, dim3((unsigned)g), dim3(128), 0, (cudaStream_t)stream, x, K, gather, expert_offsets,
                   pad_offsets, E, g_in, rows, layout, codes, sf) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}
