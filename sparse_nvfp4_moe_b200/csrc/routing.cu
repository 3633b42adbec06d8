// Routing permutation (top-k -> per-expert slot groups) and weighted combine.
//
// The grouped GEMM of the pages runs over the tokens the router sends to each
// expert (kernel line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card).  The
// slot order is (expert, token, j): a stable counting sort of the flattened
// top-k ids.  Batches of more than 1024 slots take three passes -- per-chunk
// histograms, a scan of them, and a stable scatter per 1024-slot chunk; smaller
// ones take one block and one launch.  Within a chunk match_any gives a slot's rank among
// its warp's slots of the same expert, and a [warp][expert] table of counts (up to
// 512 experts; above that the warps take turns) its place after the chunk's
// earlier warps.  Each expert's group also gets a 128-row aligned place in the
// padded GEMM operand buffers (pad_offsets).
#include "common.cuh"

#include <mutex>

namespace moesq {

constexpr int PERM_CHUNK = 1024;   // flattened (token, j) entries per block
constexpr int PERM_THREADS = 1024;

__device__ __forceinline__ int clamp_expert(int e, int E, int32_t* d_status) {
  if (e < 0 || e >= E) {
    flag(d_status, MOESQ_DFLAG_BAD_EXPERT);
    return 0;
  }
  return e;
}

// pass 1: counts[e][c] of chunk c (expert-major, so pass 2 reads rows)
__global__ void __launch_bounds__(PERM_THREADS) k_perm_count(const int32_t* __restrict__ ids,
                                                             int64_t S, int E, int nchunks,
                                                             int32_t* __restrict__ counts,
                                                             int32_t* d_status) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
  if (i < S) atomicAdd(&hist[clamp_expert(ids[i], E, d_status)], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    counts[(int64_t)e * nchunks + blockIdx.x] = hist[e];
}

// block-wide exclusive scan of one int per thread (PERM_THREADS threads)
__device__ __forceinline__ int32_t block_excl_scan(int32_t v, int32_t* warp_sums, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive
    if (lane == 31) *total = w;
  }
  __syncthreads();
  const int32_t r = x - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  __syncthreads();
  return r;
}

// pass 2 (one block): per-expert exclusive scan over chunks (in place, a warp per
// expert), then the expert offsets and their 128-row padded versions
__global__ void __launch_bounds__(PERM_THREADS) k_perm_scan(int32_t* __restrict__ counts,
                                                            int nchunks, int E,
                                                            int32_t* __restrict__ expert_offsets,
                                                            int32_t* __restrict__ pad_offsets) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t* tot = sm;  // [E]
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t total;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = warp; e < E; e += PERM_THREADS / 32) {
    int32_t* row = counts + (int64_t)e * nchunks;
    int32_t run = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 32) {
      const int c = c0 + lane;
      const int32_t v = c < nchunks ? row[c] : 0;
      int32_t x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (c < nchunks) row[c] = run + x - v;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) tot[e] = run;
  }
  __syncthreads();
  // block scan over experts: each thread owns a run of consecutive experts
  const int ept = (E + PERM_THREADS - 1) / PERM_THREADS;
  const int e0 = threadIdx.x * ept;
  int32_t la = 0, lb = 0;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      la += tot[e0 + j];
      lb += (tot[e0 + j] + 127) / 128 * 128;
    }
  int32_t ta, tb;
  int32_t ea = block_excl_scan(la, warp_sums, &total);
  ta = total;
  int32_t eb = block_excl_scan(lb, warp_sums, &total);
  tb = total;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      expert_offsets[e0 + j] = ea;
      pad_offsets[e0 + j] = eb;
      ea += tot[e0 + j];
      eb += (tot[e0 + j] + 127) / 128 * 128;
    }
  if (threadIdx.x == 0) {
    expert_offsets[E] = ta;
    pad_offsets[E] = tb;
  }
}

// pass 2 of moesq_permute, spread over the GPU: a warp per expert scans its row of
// chunk counts in place (exclusive, within the expert) and writes the expert's
// total.  Four rows of 32 chunks are in flight per warp at a time.
__global__ void __launch_bounds__(PERM_THREADS) k_perm_scan_rows(int32_t* __restrict__ counts, int nchunks,
                                                                 int E, int32_t* __restrict__ totals) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (PERM_THREADS / 32) + (threadIdx.x >> 5);
  if (e >= E) return;
  int32_t* row = counts + (int64_t)e * nchunks;
  int32_t run = 0;
  for (int c0 = 0; c0 < nchunks; c0 += 4 * 32) {
    int32_t v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u + lane;
      v[u] = c < nchunks ? row[c] : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int32_t x = v[u];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const int c = c0 + 32 * u + lane;
      if (c < nchunks) row[c] = run + x - v[u];
      run += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  if (lane == 0) totals[e] = run;
}

// Largest expert count for which a block keeps a [32 warps][E] table of per-warp
// counts in shared memory (64 KB + the run array); above it the warps take turns.
constexpr int PERM_TABLE_MAX_E = 512;
// Largest batch (flattened slots) that moesq_permute sorts in a single block: one
// chunk.  Past it three launches win, since a block loops over its 1024-slot
// sub-chunks at about 2.4 us each, while the three passes take about 8 us up to
// 16K slots.
constexpr int64_t PERM_BLOCK_MAX_S = PERM_CHUNK;

// Stable scatter of the slots [base, base + 1024) by the whole block.  run[e] is the
// next free position of expert e and is advanced past this sub-chunk's slots.  Each
// warp ranks its lanes among equal experts (match_any) and its last lane of each
// expert writes the warp's count into wcnt[warp][e]; one thread per expert then turns
// its column of counts into exclusive prefixes over the warps, which places every
// slot after all slots of lower index with the same expert.
// e: expert of this thread's slot base + threadIdx.x (any value when past S).
__device__ __forceinline__ void block_stable_scatter(int e, int64_t base, int64_t S, int k, int E, int32_t* run,
                                                     int32_t* wcnt, int32_t* __restrict__ slot_token,
                                                     int32_t* __restrict__ token_slot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = base + threadIdx.x;
  const bool valid = i < S;
  if (!valid || e < 0 || e >= E) e = 0;
  for (int x = threadIdx.x; x < 32 * E; x += blockDim.x) wcnt[x] = 0;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  const int cnt = __popc(peers);
  __syncthreads();
  if (valid && rank == cnt - 1) wcnt[warp * E + e] = cnt;
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int32_t r = run[x];
#pragma unroll
    for (int w0 = 0; w0 < 32; w0 += 16) {  // 16 loads in flight (the block's 64-register limit)
      int32_t c[16];
#pragma unroll
      for (int w = 0; w < 16; ++w) c[w] = wcnt[(w0 + w) * E + x];
#pragma unroll
      for (int w = 0; w < 16; ++w) {
        wcnt[(w0 + w) * E + x] = r;
        r += c[w];
      }
    }
    run[x] = r;
  }
  __syncthreads();
  if (valid) {
    const int pos = wcnt[warp * E + e] + rank;
    slot_token[pos] = (int32_t)(i / k);
    token_slot[i] = pos;
  }
  __syncthreads();  // wcnt and run are reused by the next sub-chunk
}

// pass 3 of moesq_permute: every block scans the expert totals itself (its own
// slot bases), block 0 also publishes the expert and padded offsets; then the
// stable scatter of the chunk, warps taking turns in order
__global__ void __launch_bounds__(PERM_THREADS) k_perm_scatter_scan(
    const int32_t* __restrict__ ids, int64_t S, int k, int E, const int32_t* __restrict__ chunk_base,
    const int32_t* __restrict__ totals, int32_t* __restrict__ expert_offsets, int32_t* __restrict__ pad_offsets,
    int32_t* __restrict__ slot_token, int32_t* __restrict__ token_slot) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t run[];  // [E] next free slot of each expert for this chunk
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t total;
  const int ept = (E + PERM_THREADS - 1) / PERM_THREADS;
  const int e0 = threadIdx.x * ept;
  int32_t la = 0, lb = 0;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      const int32_t t = totals[e0 + j];
      la += t;
      lb += (t + 127) / 128 * 128;
    }
  int32_t ea = block_excl_scan(la, warp_sums, &total);
  const int32_t ta = total;
  int32_t eb = block_excl_scan(lb, warp_sums, &total);
  const int32_t tb = total;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      const int e = e0 + j;
      const int32_t t = totals[e];
      run[e] = ea + chunk_base[(int64_t)e * gridDim.x + blockIdx.x];
      if (blockIdx.x == 0) {
        expert_offsets[e] = ea;
        pad_offsets[e] = eb;
      }
      ea += t;
      eb += (t + 127) / 128 * 128;
    }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    expert_offsets[E] = ta;
    pad_offsets[E] = tb;
  }
  __syncthreads();
  if (E <= PERM_TABLE_MAX_E) {  // table of per-warp counts after run[E] (the launch sizes it)
    const int64_t i0 = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
    block_stable_scatter(i0 < S ? ids[i0] : 0, (int64_t)blockIdx.x * PERM_CHUNK, S, k, E, run, run + E, slot_token,
                         token_slot);
    return;
  }
  const int64_t i = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
  const bool valid = i < S;
  int e = 0;
  if (valid) {
    e = ids[i];
    if (e < 0 || e >= E) e = 0;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  const int cnt = __popc(peers);
  const bool leader = valid && (rank == cnt - 1);
  for (int w = 0; w < PERM_THREADS / 32; ++w) {
    if (warp == w && valid) {
      const int pos = run[e] + rank;
      __syncwarp(vmask);
      if (leader) run[e] = pos + 1;
      slot_token[pos] = (int32_t)(i / k);
      token_slot[i] = pos;
    }
    __syncthreads();
  }
}

// moesq_permute for a batch of at most PERM_BLOCK_MAX_S slots (decode-sized): count,
// expert and padded offsets, and the stable scatter in one block and one launch
// (per-warp count table up to PERM_TABLE_MAX_E experts, else the warps take turns)
__global__ void __launch_bounds__(PERM_THREADS) k_perm_block(const int32_t* __restrict__ ids, int64_t S, int k,
                                                             int E, int32_t* __restrict__ expert_offsets,
                                                             int32_t* __restrict__ pad_offsets,
                                                             int32_t* __restrict__ slot_token,
                                                             int32_t* __restrict__ token_slot, int32_t* d_status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm_block[];
  int32_t* hist = sm_block;      // [E] counts, then the next free slot of each expert
  int32_t* wcnt = sm_block + E;  // [32][E] per-warp counts of a sub-chunk (table form only)
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t total;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  // every thread keeps the experts of its slots (threadIdx.x + 1024 j) for the scatter
  int ev[PERM_BLOCK_MAX_S / PERM_THREADS];
#pragma unroll
  for (int j = 0; j < PERM_BLOCK_MAX_S / PERM_THREADS; ++j) {
    const int64_t i = threadIdx.x + (int64_t)PERM_THREADS * j;
    ev[j] = i < S ? clamp_expert(ids[i], E, d_status) : 0;
  }
#pragma unroll
  for (int j = 0; j < PERM_BLOCK_MAX_S / PERM_THREADS; ++j)
    if (threadIdx.x + (int64_t)PERM_THREADS * j < S) atomicAdd(&hist[ev[j]], 1);
  __syncthreads();
  const int ept = (E + PERM_THREADS - 1) / PERM_THREADS;
  const int e0 = threadIdx.x * ept;
  int32_t la = 0, lb = 0;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      la += hist[e0 + j];
      lb += (hist[e0 + j] + 127) / 128 * 128;
    }
  int32_t ea = block_excl_scan(la, warp_sums, &total);
  const int32_t ta = total;
  int32_t eb = block_excl_scan(lb, warp_sums, &total);
  const int32_t tb = total;
  for (int j = 0; j < ept; ++j)
    if (e0 + j < E) {
      const int32_t c = hist[e0 + j];
      expert_offsets[e0 + j] = ea;
      pad_offsets[e0 + j] = eb;
      hist[e0 + j] = ea;  // each thread rewrites only its own experts
      ea += c;
      eb += (c + 127) / 128 * 128;
    }
  if (threadIdx.x == 0) {
    expert_offsets[E] = ta;
    pad_offsets[E] = tb;
  }
  __syncthreads();
  if (E <= PERM_TABLE_MAX_E) {
#pragma unroll
    for (int j = 0; j < PERM_BLOCK_MAX_S / PERM_THREADS; ++j)
      if ((int64_t)PERM_THREADS * j < S)
        block_stable_scatter(ev[j], (int64_t)PERM_THREADS * j, S, k, E, hist, wcnt, slot_token, token_slot);
    return;
  }
  static_assert(PERM_BLOCK_MAX_S == PERM_THREADS, "the turns form scatters one chunk");
  const int64_t i = threadIdx.x;
  const bool valid = i < S;
  const int e = ev[0];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  const int cnt = __popc(peers);
  const bool leader = valid && (rank == cnt - 1);
  for (int w = 0; w < PERM_THREADS / 32; ++w) {
    if (warp == w && valid) {
      const int pos = hist[e] + rank;
      __syncwarp(vmask);
      if (leader) hist[e] = pos + 1;
      slot_token[pos] = (int32_t)(i / k);
      token_slot[i] = pos;
    }
    __syncthreads();
  }
}

// pass 3: stable scatter; warps of the chunk take turns in order
__global__ void __launch_bounds__(PERM_THREADS) k_perm_scatter(
    const int32_t* __restrict__ ids, int64_t S, int k, int E, const int32_t* __restrict__ chunk_base,
    const int32_t* __restrict__ expert_offsets, int32_t* __restrict__ slot_token,
    int32_t* __restrict__ token_slot) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  extern __shared__ int32_t run[];  // [E] next free slot of each expert for this chunk
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    run[e] = expert_offsets[e] + chunk_base[(int64_t)e * gridDim.x + blockIdx.x];
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * PERM_CHUNK + threadIdx.x;
  const bool valid = i < S;
  int e = 0;
  if (valid) {
    e = ids[i];
    if (e < 0 || e >= E) e = 0;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  const int cnt = __popc(peers);
  const bool leader = valid && (rank == cnt - 1);
  for (int w = 0; w < PERM_THREADS / 32; ++w) {
    if (warp == w && valid) {
      const int pos = run[e] + rank;
      __syncwarp(vmask);
      if (leader) run[e] = pos + 1;
      slot_token[pos] = (int32_t)(i / k);
      token_slot[i] = pos;
    }
    __syncthreads();
  }
}

// combine: thread per (token, 8 features); float32 in j order, no fused multiply-add
template <bool BATCHED>
__global__ void k_unpermute(const uint16_t* __restrict__ y, const int32_t* __restrict__ token_slot,
                            const float* __restrict__ topk_w, int64_t T, int k, int64_t H,
                            uint16_t* __restrict__ out) {
  pdl_wait();  // the previous kernel's outputs are complete past here
  pdl_trigger();
  const int64_t vec = H / 8;
  const int64_t n = T * vec;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vec, c = i % vec;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
    if constexpr (!BATCHED) {
      // large batches: one slot at a time (fewer registers, more warps to hide latency)
      for (int j = 0; j < k; ++j) {
        const int64_t s = token_slot[t * k + j];
        const float w = topk_w[t * k + j];
        const uint4 u = *reinterpret_cast<const uint4*>(y + s * H + 8 * c);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(w, bf16_bits_to_float(wd[q] & 0xFFFF)));
          acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(w, bf16_bits_to_float(wd[q] >> 16)));
        }
      }
    } else {
      // slots in chunks of 8: the slot indices, weights and rows of a chunk are loaded
      // before the sums, which still run in j order
      for (int j0 = 0; j0 < k; j0 += 8) {
        int64_t sv[8];
        float wv[8];
        uint4 uv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          sv[u] = j < k ? (int64_t)token_slot[t * k + j] : -1;
          wv[u] = j < k ? topk_w[t * k + j] : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          uv[u] = sv[u] >= 0 ? *reinterpret_cast<const uint4*>(y + sv[u] * H + 8 * c) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u < k) {
            const float w = wv[u];
            const uint32_t wd[4] = {uv[u].x, uv[u].y, uv[u].z, uv[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(w, bf16_bits_to_float(wd[q] & 0xFFFF)));
              acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(w, bf16_bits_to_float(wd[q] >> 16)));
            }
          }
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = float_to_bf16_bits(acc[2 * q]) | (float_to_bf16_bits(acc[2 * q + 1]) << 16);
    *reinterpret_cast<uint4*>(out + t * H + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace moesq

using namespace moesq;

// dynamic shared memory above the 48 KB default needs the kernel's opt-in
template <typename Kernel>
static cudaError_t allow_dynamic_smem(Kernel kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute((const void*)kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

extern "C" int64_t moesq_padded_rows(int64_t S, int32_t E) {
  if (S < 0 || E <= 0) return 0;
  const int64_t extra = 127 * (int64_t)(S < E ? S : E);  // only nonempty groups pad
  return (S + extra + 127) / 128 * 128;
}

extern "C" moesq_status moesq_permute_workspace_size(int64_t T, int32_t k, int32_t E,
                                                     size_t* bytes) {
  MOESQ_REQUIRE(bytes && T >= 0 && k >= 1 && k <= 32 && E >= 1 && E <= 4096,
                MOESQ_ERR_INVALID_ARG);
  const int64_t S = T * k;
  const int64_t nchunks = (S + PERM_CHUNK - 1) / PERM_CHUNK;
  // per-chunk expert counts, then one total per expert
  *bytes = (size_t)((nchunks > 0 ? nchunks : 1) * E + E) * sizeof(int32_t);
  return MOESQ_OK;
}

extern "C" moesq_status moesq_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E,
                                      int32_t* expert_offsets, int32_t* pad_offsets,
                                      int32_t* slot_token, int32_t* token_slot, void* ws,
                                      size_t ws_bytes, int32_t* d_status, moesq_stream_t stream) {
  MOESQ_REQUIRE(expert_offsets && pad_offsets, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(T >= 0 && k >= 1 && k <= 32 && E >= 1 && E <= 4096, MOESQ_ERR_INVALID_ARG);
  const int64_t S = T * k;
  MOESQ_REQUIRE(S < (1ll << 31), MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(S == 0 || (topk_ids && slot_token && token_slot), MOESQ_ERR_INVALID_ARG);
  size_t need = 0;
  moesq_permute_workspace_size(T, k, E, &need);
  MOESQ_REQUIRE(ws && ws_bytes >= need, MOESQ_ERR_WORKSPACE);
  cudaStream_t s = (cudaStream_t)stream;
  const int nchunks = (int)((S + PERM_CHUNK - 1) / PERM_CHUNK);
  int32_t* counts = (int32_t*)ws;
  const size_t shm = (size_t)E * sizeof(int32_t);
  if (nchunks == 0) {  // no slots: the offsets are all zero
    if (moesq_launch(k_perm_scan, dim3(1), dim3(PERM_THREADS), shm, s, counts, nchunks, E, expert_offsets,
                     pad_offsets) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    return MOESQ_OK;
  }
  const bool table = E <= PERM_TABLE_MAX_E;
  const size_t shm_table = (size_t)33 * E * sizeof(int32_t);  // run[E] + per-warp counts [32][E]
  if (S <= PERM_BLOCK_MAX_S) {  // decode-sized: everything in one block and one launch
    const size_t shm_block = table ? shm_table : shm;
    if (allow_dynamic_smem(k_perm_block, shm_block) != cudaSuccess) return MOESQ_ERR_CUDA;
    if (moesq_launch(k_perm_block, dim3(1), dim3(PERM_THREADS), shm_block, s, topk_ids, S, k, E, expert_offsets,
                     pad_offsets, slot_token, token_slot, d_status) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    return MOESQ_OK;
  }
  int32_t* totals = counts + (int64_t)nchunks * E;
  if (moesq_launch(k_perm_count, dim3(nchunks), dim3(PERM_THREADS), shm, s, topk_ids, S, E, nchunks, counts,
                   d_status) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  if (moesq_launch(k_perm_scan_rows, dim3((E + PERM_THREADS / 32 - 1) / (PERM_THREADS / 32)), dim3(PERM_THREADS),
                   0, s, counts, nchunks, E, totals) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  const size_t shm_scatter = table ? shm_table : shm;
  if (allow_dynamic_smem(k_perm_scatter_scan, shm_scatter) != cudaSuccess) return MOESQ_ERR_CUDA;
  if (moesq_launch(k_perm_scatter_scan, dim3(nchunks), dim3(PERM_THREADS), shm_scatter, s, topk_ids, S, k, E,
                   (const int32_t*)counts, (const int32_t*)totals, expert_offsets, pad_offsets, slot_token,
                   token_slot) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_unpermute(const uint16_t* y, const int32_t* token_slot,
                                        const float* topk_w, int64_t T, int32_t k, int64_t H,
                                        uint16_t* out, moesq_stream_t stream) {
  MOESQ_REQUIRE(T >= 0 && k >= 1 && H >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(H % 8 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (T == 0 || H == 0) return MOESQ_OK;
  MOESQ_REQUIRE(y && token_slot && topk_w && out, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(y) && moesq_aligned16(out), MOESQ_ERR_INVALID_ARG);
  const int64_t n = T * (H / 8);
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  // small batches (decode): every slot's loads in flight at once; large: more warps
  const cudaError_t err =
      T <= 512 ? moesq_launch(k_unpermute<true>, dim3((unsigned)g), dim3(256), 0, (cudaStream_t)stream, y, token_slot,
                              topk_w, T, k, H, out)
               : moesq_launch(k_unpermute<false>, dim3((unsigned)g), dim3(256), 0, (cudaStream_t)stream, y, token_slot,
                              topk_w, T, k, H, out);
  if (err != cudaSuccess) return MOESQ_ERR_CUDA;
  return MOESQ_OK;
}

// ---------------------------------------------------------------------------
// moesq_permute_noalloc: moesq_permute for callers that cannot allocate.
//
// Its only scratch (the per-chunk expert counts) lives in a fixed file-scope
// device array, so the caller passes inputs and outputs only.  Every GPU that
// loads this library keeps the array (1 MiB) until the process exits.  All calls
// share it: calls whose executions overlap on the GPU (different streams, or
// different host threads on one device) race on it and must be serialised by
// the caller.  Every word a call reads is first written by that same call, so
// nothing needs clearing between calls.
static __device__ __align__(256) int32_t g_perm_noalloc_scratch[MOESQ_PERMUTE_NOALLOC_MAX_COUNTS];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
int32_t* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
moesq_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOESQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOESQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_perm_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return MOESQ_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = (int32_t*)p;
  }
  *out = g_noalloc_ptr[dev];
  return MOESQ_OK;
}
}  // namespace

extern "C" moesq_status moesq_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k,
                                              int32_t E, int32_t* expert_offsets,
                                              int32_t* pad_offsets, int32_t* slot_token,
                                              int32_t* token_slot, int32_t* d_status,
                                              moesq_stream_t stream) {
  MOESQ_REQUIRE(expert_offsets && pad_offsets, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(T >= 0 && k >= 1 && k <= 32 && E >= 1 && E <= 4096, MOESQ_ERR_INVALID_ARG);
  const int64_t S = T * k;
  MOESQ_REQUIRE(S < (1ll << 31), MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(S == 0 || (topk_ids && slot_token && token_slot), MOESQ_ERR_INVALID_ARG);
  const int64_t nchunks = (S + PERM_CHUNK - 1) / PERM_CHUNK;
  MOESQ_REQUIRE(nchunks * E <= MOESQ_PERMUTE_NOALLOC_MAX_COUNTS, MOESQ_ERR_CAPACITY);
  int32_t* counts = nullptr;
  const moesq_status st = noalloc_scratch(&counts);
  if (st != MOESQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t shm = (size_t)E * sizeof(int32_t);
  if (nchunks > 0) {
    k_perm_count<<<(int)nchunks, PERM_THREADS, shm, s>>>(topk_ids, S, E, (int)nchunks, counts,
                                                        d_status);
    MOESQ_CHECK_LAUNCH();
  }
  k_perm_scan<<<1, PERM_THREADS, shm, s>>>(counts, (int)nchunks, E, expert_offsets, pad_offsets);
  MOESQ_CHECK_LAUNCH();
  if (nchunks > 0) {
    k_perm_scatter<<<(int)nchunks, PERM_THREADS, shm, s>>>(topk_ids, S, k, E, counts,
                                                           expert_offsets, slot_token, token_slot);
    MOESQ_CHECK_LAUNCH();
  }
  return MOESQ_OK;
}
