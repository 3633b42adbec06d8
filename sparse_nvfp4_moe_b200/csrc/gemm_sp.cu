// Grouped paired-4:8 sparse NVFP4 GEMM on the sm_100a tensor cores.
//
// The pages' kernel is a "paired-4:8 sparse NVFP4 grouped GEMM" for SM100
// (header list of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; "Kernels" of
// the MoESQ repository README).  The scale group is 32 dense K because the
// Blackwell sparse NVFP4 MMA takes one scale per 32 dense K = 16 kept values
// ("Compression details", same card).  This kernel:
//
//   * puts the weights on the sparse operand A of tcgen05.mma.sp and the routed
//     tokens of one expert on B (N <= 128), so the compressed weight bytes are
//     the streamed operand and the weight values are read exactly as stored
//     (weight_sparse_packed is the compressed A operand: kept elements in K order);
//   * runs on CTA pairs (clusters of 2 on two SMs, cta_group::2): one MMA covers
//     256 weight rows, 128 per CTA, and each CTA stages only half of the token
//     tile, which halves the token bytes every SM loads and reads per MMA (the
//     shared-memory operand reads bound a single-CTA sparse MMA);
//   * is persistent: each pair walks a static list of (expert, token tile,
//     weight-tile pair) work items built on the device from the routing
//     offsets, so empty experts cost nothing;
//   * is warp-specialised: warp 0 of each CTA issues the TMA copies (values,
//     tokens, metadata, block scales) into a 4-stage shared-memory ring of
//     512-deep K blocks; warp 1 of the first CTA copies metadata and scales
//     smem->TMEM (tcgen05.cp) and issues the MMAs (dense K = 128 each, four per
//     stage); warps 2..17 of each CTA drain its double-buffered FP32
//     accumulators (tcgen05.ld) while the next tile runs;
//   * reads weight tiles whose rows the repack interleaves, so that one 16x256b
//     TMEM load gives a thread both operands of an epilogue pair (gate and up of
//     an output, or two neighbouring outputs) and no lanes exchange values;
//   * fuses the epilogue: FP32 or bf16 output per slot, or SwiGLU followed by
//     NVFP4 requantisation written straight into the next GEMM's B operand
//     layout (codes + 512-byte scale blocks);
//   * on large batches runs the SwiGLU GEMM on wide items: two token tiles of an
//     expert per item, one MMA of N <= 256 per K step, so the weight tile is read
//     from shared memory once per 256 tokens (accumulators of consecutive items
//     overlap in TMEM, see namespace wide);
//   * on decode-sized batches takes each item's expert from a per-pair table built at
//     set-up instead of searching the expert records item after item;
//   * optionally fuses the weighted combine into the down GEMM's epilogue (a
//     deterministic arrival count per token and output tile; slower than the
//     separate combine, see moesq_grouped_gemm_down_combine).
//
// The same kernel, with a dense stage geometry (256-deep stages of four dense
// kind::mxf4nvf4 MMAs, no metadata), is the dense comparison GEMM on decoded
// weights (moesq_grouped_gemm_dense).
//
// Every mbarrier wait is bounded (2 s); on expiry the kernel flags
// MOESQ_DFLAG_TIMEOUT, drains its own copies in flight, frees TMEM and exits.
#include "common.cuh"

#include <atomic>
#include <mutex>

namespace moesq {
namespace sp {

constexpr int BM = 128;           // weight rows per tile
constexpr int BN = 128;           // max tokens per tile
constexpr int B_CHUNK = (BN / 2) * 128;    // this CTA's half of the tokens, 256 dense K: 128 B per row (SW128)
constexpr int SF_BYTES = 4 * 512;          // one 512-byte scale block per MMA and operand, four MMAs a stage
constexpr int MAX_STAGES = 5;
// Stage geometry.  Every copy instruction costs the single issuing thread about the
// same whatever its size, so a stage is moved by few, large copies: one for the
// weight tile, one or two for the token tile, one each for metadata and the two
// scale blocks.
//   sparse: 512 dense K a stage, four sparse MMAs of 128 dense K (one scale per 32)
//   dense (the comparison kernel on decoded weights): 256 dense K a stage, four
//   dense MMAs of 64 dense K (one scale per 16, the 32-group scales duplicated)
template <bool DENSE> struct Geo;
template <> struct Geo<false> {
  static constexpr int BK = 512, KMMA = 128, STAGES = 4;
  static constexpr int A_BYTES = BM * BK / 4;  // compressed values: 128 B per row (SW128)
  static constexpr int B_BYTES = 2 * B_CHUNK;  // two 256-deep token chunks
  static constexpr int E_BYTES = 2 * BM * 16;  // metadata: 16 B per row per 256 dense K
};
template <> struct Geo<true> {
  static constexpr int BK = 256, KMMA = 64, STAGES = 5;
  static constexpr int A_BYTES = BM * BK / 2;  // dense codes: 128 B per row (SW128)
  static constexpr int B_BYTES = B_CHUNK;      // one 256-deep token chunk
  static constexpr int E_BYTES = 0;
};
template <bool DENSE>
__host__ __device__ constexpr int stage_bytes() {
  return Geo<DENSE>::A_BYTES + Geo<DENSE>::B_BYTES + Geo<DENSE>::E_BYTES + 2 * SF_BYTES;  // 40960 / 28672
}
constexpr int EPI_BYTES = 32768;  // epilogue space: bf16 staging, f32 transposes, SwiGLU amax swaps
constexpr int MAX_E = 1024;
constexpr int ITEM_TAB = 128;  // work items per pair whose expert is looked up, not searched
// Sixteen epilogue warps, four per sub-partition: the epilogue is bound by issue
// and latency (TMEM loads, MUFU-heavy SiLU, lane exchanges), so it wants warps;
// the 18 warps are allocated as 20, which leaves 96 registers a thread.
constexpr int EPI_WARPS = 16;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int THREADS = 64 + EPI_THREADS;  // producer warp, MMA warp, epilogue warps
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0, TM_E = 256, TM_SFA = 264, TM_SFB = 280;
// Wide items (the SwiGLU gate_up GEMM on large batches): a work item is one weight-tile
// pair and two 128-token tiles of an expert, and each 128-deep step is ONE MMA with
// N = 256, so the weight tile is read from shared memory once for 256 tokens: a stage
// moves 58 KB into each SM (weights 22 KB, the CTA's 128 token rows 32 KB, the two
// 128-row token scale blocks 4 KB) and its MMAs read 48 KB, against 80 KB of copies
// and reads for the same work in two one-tile items.  Two 256-column accumulators do
// not fit in TMEM beside the metadata and scales, so the accumulators of consecutive
// items overlap: items alternate between columns 0-255 and 128-383, and the next item's
// MMAs start as soon as the epilogue has read the shared columns 128-255 (one token
// tile), while the other tile's columns stay untouched until the item after it.
namespace wide {
constexpr int STAGES = 3;
constexpr int A_BYTES = Geo<false>::A_BYTES, E_BYTES = Geo<false>::E_BYTES;
constexpr int B_CHUNK = BN * 128;  // 128 token rows of one 256-deep chunk (SW128)
constexpr int B_BYTES = 2 * B_CHUNK;
constexpr int OFF_E = A_BYTES + B_BYTES, OFF_SFA = OFF_E + E_BYTES, OFF_SFB = OFF_SFA + SF_BYTES;
constexpr int STAGE_BYTES = OFF_SFB + 2 * SF_BYTES;  // 59392
constexpr int EPI_BYTES = 4096;                      // the SwiGLU epilogue's amax swaps and code multipliers
constexpr uint32_t TM_E = 384, TM_SFA = 392, TM_SFB = 408;  // SFB: 8 columns per MMA (token rows 0-127, 128-255)
static_assert(TM_SFB + 32 <= TMEM_COLS && STAGE_BYTES % 1024 == 0, "wide geometry");
}  // namespace wide

// The down GEMM with the weighted combine fused into its epilogue (see the bf16
// epilogue): a template value of its own, not an `epilogue` argument of the C ABI.
constexpr int EPI_BF16_COMBINE = 3;

struct Params {
  const uint8_t* meta;
  const uint8_t* sfw;
  const float* alpha_w;
  const uint8_t* act_sf;
  const float* g_act;
  const int32_t* expert_offsets;
  const int32_t* pad_offsets;
  const float* g_next;
  void* out;
  uint8_t* out_sf;
  int32_t* d_status;
  int E, M, K, epi, gate_up;
  int exact;  // gate_up with its own up global: alpha_w is [E, 2] (gate, up)
  int64_t S, P_cap;
  // EPI_BF16_COMBINE only: routing, weights, per-(token, 128-output tile) arrival counts
  // (zero at launch), the combined output [T, M] bf16; p.out is the per-slot y
  const int32_t* slot_token;
  const int32_t* token_slot;
  const float* topk_w;
  int32_t* arrivals;
  uint16_t* comb_out;
  int k;
};

struct Smem {
  // SwiGLU epilogue staging, double-buffered over tiles: per 32-token column block
  // the requantised codes (32 B = 64 features per token) and the scale pairs
  alignas(128) uint8_t hstg[2][4][32][32];
  alignas(16) uint8_t sstg[2][4][32][2];
  // full[s]: stage s landed.  empty[s]: stage s consumed by the tensor core.
  uint64_t full[MAX_STAGES], empty[MAX_STAGES], acc_full[2], acc_empty[2], done;
  uint32_t tmem_base;
  int abort;
  // per-expert tables, read from global memory once at set-up so that no role
  // waits on a global load between tiles.  One 16-byte record per expert, so
  // that a role finds everything about its next tile in one shared load:
  // {end of its token tiles (prefix sum), first routed slot, first padded row,
  // routed-slot count}
  int4 rec[MAX_E];
  float2 ag[MAX_E];  // {g_act[e] * alpha_w[e] (the accumulator's scale), global scale of the requantised output}
  // the expert of each of this pair's work items when the pair has at most ITEM_TAB of
  // them (decode-sized batches, where every item jumps over several experts), found at
  // set-up by the prefix-sum warp; n_tab = 0: the roles walk (see TileWalk)
  uint16_t item_e[ITEM_TAB];
  int n_tab;
};

template <bool DENSE>
constexpr size_t smem_bytes() {
  return 1024 /*align*/ + (size_t)Geo<DENSE>::STAGES * stage_bytes<DENSE>() + EPI_BYTES + sizeof(Smem);
}
constexpr size_t smem_bytes_wide() {
  return 1024 /*align*/ + (size_t)wide::STAGES * wide::STAGE_BYTES + wide::EPI_BYTES + sizeof(Smem);
}
static_assert(smem_bytes<false>() <= 227 * 1024 && smem_bytes<true>() <= 227 * 1024 &&
                  smem_bytes_wide() <= 227 * 1024,
              "shared memory budget");
static_assert(Geo<false>::STAGES <= MAX_STAGES && Geo<true>::STAGES <= MAX_STAGES, "barrier arrays");

template <bool DENSE>
__device__ __forceinline__ uint32_t make_idesc(uint32_t n) {
  return (DENSE ? 0u : 1u << 2)  // sparse
         | (1u << 7)          // A: E2M1
         | (1u << 10)         // B: E2M1
         | ((n >> 3) << 17)   // N
         | (0u << 23)         // scale factors UE4M3
         | ((uint32_t)(2 * BM >> 4) << 24);  // M = 256 over the CTA pair
}

struct Tile {
  int e, nt, mt, n_rows;
  int n_rows1;  // wide items: tokens of the second 128-token tile (0: none)
  int prow;  // first padded row of the token tile
  int s0;    // first routed slot of the token tile
};

// Work items run over (token tile q, weight-tile pair m), m fastest; pair `pid`
// of `npairs` takes items pid, pid + npairs, ...  Every role walks its items in
// that order, stepping (q, m) by a precomputed (dq, dm) and the expert forward
// from the previous item's, so no role divides or searches between tiles.  The
// current expert's record is kept in registers and the next expert's is loaded
// as soon as the walk enters an expert, so the shared-memory load is consumed a
// tile later (its latency is hidden behind the tile's work).
struct TileWalk {
  int q, m, dq, dm, e;
  int j, ntab;    // item index of this pair; items with j < ntab take their expert from item_e
  int4 cur, nxt;  // rec[e], rec[e + 1] (rec[e] again past the last expert)
  __device__ __forceinline__ TileWalk(const Smem& s, int pid, int npairs, int MT2, int E)
      : q(pid / MT2), m(pid % MT2), dq(npairs / MT2), dm(npairs % MT2), e(0), j(0), ntab(s.n_tab) {
    cur = s.rec[0];
    nxt = E > 1 ? s.rec[1] : cur;
  }
  __device__ __forceinline__ void advance(int MT2) {
    ++j;
    m += dm;
    q += dq;
    if (m >= MT2) {
      m -= MT2;
      ++q;
    }
  }
};

// The current item of `w`: its expert from the set-up table when the pair has one
// (decode-sized batches), else by the walk.  Empty experts end their tiles where they
// start; when the next expert does not hold tile q either, a binary search over the
// tile-end prefix sums finds the first expert that does, so a walk over thousands of
// empty experts costs log2(E) loads, not E.
template <int NT = 1>
__device__ __forceinline__ Tile decode_tile(const Smem& s, TileWalk& w, int E) {
  if (NT == 1 && w.j < w.ntab) {  // the same for every item of the pair: table or walk
    const int e = s.item_e[w.j];
    if (e != w.e) {
      w.e = e;
      w.cur = s.rec[e];
    }
  } else if (w.cur.x <= w.q && w.e + 1 < E) {
    if (w.nxt.x > w.q) {
      ++w.e;
      w.cur = w.nxt;
    } else {
      // rec[e + 1].x <= q < rec[E - 1].x (q is below the total tile count)
      int lo = w.e + 2, hi = E - 1;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s.rec[mid].x > w.q) hi = mid;
        else lo = mid + 1;
      }
      w.e = lo;
      w.cur = s.rec[lo];
    }
    w.nxt = w.e + 1 < E ? s.rec[w.e + 1] : w.cur;
  }
  const int4 r = w.cur;
  Tile t;
  t.e = w.e;
  t.mt = w.m;
  t.nt = w.q - (r.x - (r.w + NT * BN - 1) / (NT * BN));
  const int rem = r.w - t.nt * (NT * BN);
  t.n_rows = rem < BN ? rem : BN;
  t.n_rows1 = NT == 2 ? (rem - BN < 0 ? 0 : (rem - BN < BN ? rem - BN : BN)) : 0;
  t.prow = r.z + t.nt * (NT * BN);
  t.s0 = r.y + t.nt * (NT * BN);
  return t;
}

// bounded wait used only while draining at exit: ignores the abort flag
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

template <int EPI, bool DENSE, int NT = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_grouped_gemm_sp(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_b16, const __grid_constant__ CUtensorMap tmap_e,
                      const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                      const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_b_3d,
                      const Params p) {
  using G = Geo<DENSE>;
  static_assert(NT == 1 || (NT == 2 && !DENSE && EPI == MOESQ_EPI_SWIGLU_NVFP4), "wide items: SwiGLU gate_up");
  constexpr int STAGES = NT == 2 ? wide::STAGES : G::STAGES;
  constexpr int STAGE_BYTES = NT == 2 ? wide::STAGE_BYTES : stage_bytes<DENSE>();
  constexpr int A_BYTES = G::A_BYTES, B_BYTES = NT == 2 ? wide::B_BYTES : G::B_BYTES, E_BYTES = G::E_BYTES;
  constexpr int EPI_SPACE = NT == 2 ? wide::EPI_BYTES : EPI_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* epi = (float*)(smem + STAGES * STAGE_BYTES);
  Smem& S = *(Smem*)(smem + STAGES * STAGE_BYTES + EPI_SPACE);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the pair's MMAs
  const bool lead = rank == 0;
  const int E = p.E, MT = p.M / BM, MT2 = (MT + 1) / 2;
  // K stages, MMAs over K (= scale blocks per 128 rows), 256-deep metadata chunks
  const int nkb = (p.K + G::BK - 1) / G::BK, kb128 = p.K / G::KMMA, nkb256 = (p.K + 255) / 256;
  const int32_t* off = p.expert_offsets;
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  // ---- set-up: barriers, tables, TMEM (both CTAs), then a cluster barrier so
  // that no CTA signals a barrier of its peer before the peer initialised it
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&S.full[i], 1);   // used in CTA 0: its producer's arrival + both CTAs' bytes
      mbar_init(&S.empty[i], 1);  // one multicast commit per use, in both CTAs
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.acc_full[i], 1);
      mbar_init(&S.acc_empty[i], 2 * EPI_WARPS);  // used in CTA 0: every epilogue warp of the pair
    }
    mbar_init(&S.done, 1);
    S.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
    tma_prefetch_desc(&tmap_b16);
    tma_prefetch_desc(&tmap_e);
    tma_prefetch_desc(&tmap_sfa);
    tma_prefetch_desc(&tmap_sfb);
    tma_prefetch_desc(&tmap_b_3d);
  }
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  // everything above is independent of the inputs; the routing offsets and the
  // activations are written by the kernels before this one
  pdl_wait();
  pdl_trigger();
  // per-expert tables: one round of parallel global loads
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int o0 = off[e], o1 = off[e + 1];
    S.rec[e] = make_int4(0, o0, p.pad_offsets[e], o1 - o0);
    S.ag[e] = make_float2(__fmul_rn(p.g_act[e], p.alpha_w[p.exact ? 2 * e : e]), p.g_next ? p.g_next[e] : 0.0f);
  }
  __syncthreads();
  if (warp == 0) {  // end of expert e's token tiles = sum over e' <= e of ceil(T_e' / BN)
    int run = 0, nz = 0;  // tiles, experts that hold any
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int v = 0;
      if (e < E) v = (S.rec[e].w + NT * BN - 1) / (NT * BN);
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (e < E) S.rec[e].x = run + x;
      run += __shfl_sync(0xffffffffu, x, 31);
      nz += __popc(__ballot_sync(0xffffffffu, v > 0));
    }
    // decode-sized batches: the expert of each of this pair's items, one binary search
    // per item by the lanes of this warp.  Used where a role's walk, which advances
    // npairs / MT2 tiles an item, would jump over two or more experts an item on
    // average and so search item after item; elsewhere the walk steps through the
    // records it holds, which costs less than a table load.  Wide items run on large
    // batches only.
    __syncwarp();
    const int tot = run * MT2, dq = npairs / MT2;
    const int mine = pair_id < tot ? (tot - 1 - pair_id) / npairs + 1 : 0;
    const int ntab = NT == 1 && mine >= 2 && mine <= ITEM_TAB && 2 * run < dq * nz ? mine : 0;
    for (int j = lane; j < ntab; j += 32) {
      const int qj = (pair_id + j * npairs) / MT2;
      int lo = 0, hi = E - 1;  // the first expert whose tile end exceeds qj
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (S.rec[mid].x > qj) hi = mid;
        else lo = mid + 1;
      }
      S.item_e[j] = (uint16_t)lo;
    }
    if (lane == 0) S.n_tab = ntab;
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const int total = S.rec[E - 1].x * MT2;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ================================================================ producer
    // Both CTAs load their own weight rows, their half of the token rows and the
    // full token scale block into their own shared memory; every copy completes
    // on CTA 0's full barrier, where CTA 0 posts the pair's byte count.
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      long fills = 0;
      TileWalk walk(S, pair_id, npairs, MT2, E);
      uint32_t full_lead[STAGES];
#pragma unroll
      for (int i = 0; i < STAGES; ++i) full_lead[i] = cluster_map(&S.full[i], 0);
      const bool b3d = !DENSE && (p.K % 256) == 0;  // both 256-deep token chunks of a stage in one 3-D box
      for (int id = pair_id; id < total; id += npairs, walk.advance(MT2)) {
        const Tile t = decode_tile<NT>(S, walk, E);
        const int mt = min(2 * t.mt + (int)rank, MT - 1);  // an odd last tile is loaded twice
        int prow = t.prow;
        if (prow < 0 || (int64_t)prow + BN > p.P_cap) {  // inconsistent offsets: stay in bounds
          flag(p.d_status, MOESQ_DFLAG_CAPACITY);
          prow = 0;
        }
        const int n_mma = max(16, (t.n_rows + (NT == 2 ? t.n_rows1 : 0) + 15) / 16 * 16);
        const int brow = prow + (int)rank * (n_mma / 2);  // this CTA's half of the token rows
        const int wt = t.e * MT + mt;                   // weight tile
        // a tile of <= 32 tokens loads 16-row B boxes (decode-sized groups)
        const bool small = n_mma <= 32;
        const void* tb = small ? (const void*)&tmap_b16 : (const void*)&tmap_b;
        const void* tb3 = &tmap_b_3d;
        const uint32_t b_box = small ? 16 * 128 : B_CHUNK;
        // wide items holding two token tiles: this CTA's (up to) 128 token rows of both
        // 256-deep chunks in one 3-D box of 128 rows, and the second tile's scale block
        const bool two = NT == 2 && t.n_rows1 > 0;
        for (int kb = 0; kb < nkb; ++kb) {
          mbar_wait_spin(&S.empty[stage], phase ^ 1, abort, p.d_status);
          const int nk = min(4, kb128 - 4 * kb);  // 128-deep MMAs in this stage
          const int nc = DENSE ? 1 : (nk + 1) >> 1;  // 256-deep token chunks in this stage
          uint8_t* st = smem + stage * STAGE_BYTES;
          uint32_t bar = full_lead[0];
#pragma unroll
          for (int i = 1; i < STAGES; ++i)
            if (stage == i) bar = full_lead[i];
          if constexpr (NT == 2) {
            if (lead)
              mbar_arrive_expect_tx(&S.full[stage], two ? 2u * (A_BYTES + B_BYTES + E_BYTES + 3 * SF_BYTES)
                                                        : 2u * (A_BYTES + nc * b_box + E_BYTES + 2 * SF_BYTES));
          } else {
            if (lead) mbar_arrive_expect_tx(&S.full[stage], 2u * (A_BYTES + nc * b_box + E_BYTES + 2 * SF_BYTES));
          }
          // weight tile in the repack's interleaved row order: gate and up rows of
          // outputs 64mt..64mt+63 in one 5-D box (byte, j, gate/up, h, 16-row group), or
          // down rows 128mt.. in one 4-D box (byte, j, p, 16-row group)
          if (p.gate_up) tma_load_5d_pair(st, &tmap_a, kb * 128, 0, 0, 0, t.e * (p.M / 16) + 4 * mt, bar);
          else tma_load_4d_pair(st, &tmap_a, kb * 128, 0, 0, (t.e * p.M + BM * mt) / 16, bar);
          if constexpr (NT == 2) {  // chunk 1 lands at wide::B_CHUNK (K % 512 == 0: nc == 2)
            if (two) {
              tma_load_3d_pair(st + A_BYTES, tb3, 0, brow, 2 * kb, bar);
            } else {
              tma_load_2d_pair(st + A_BYTES, tb, kb * 256, brow, bar);
              tma_load_2d_pair(st + A_BYTES + wide::B_CHUNK, tb, kb * 256 + 128, brow, bar);
            }
          } else if (b3d && nc > 1 && !small) {  // 64-row chunks: chunk 1 lands at B_CHUNK as the MMA expects
            tma_load_3d_pair(st + A_BYTES, tb3, 0, brow, 2 * kb, bar);
          } else {
            tma_load_2d_pair(st + A_BYTES, tb, kb * (G::BK / 2), brow, bar);
            if (nc > 1) tma_load_2d_pair(st + A_BYTES + B_CHUNK, tb, kb * 256 + 128, brow, bar);
          }
          // metadata (2 KB per 256 dense K) and scale blocks (512 B per 128 dense K)
          // as 256-byte rows; a stage always moves 4 KB + 2 KB + 2 KB
          if constexpr (!DENSE) tma_load_2d_pair(st + A_BYTES + B_BYTES, &tmap_e, 0, (wt * nkb256 + 2 * kb) * 8, bar);
          tma_load_2d_pair(st + A_BYTES + B_BYTES + E_BYTES, &tmap_sfa, 0, (wt * kb128 + 4 * kb) * 2, bar);
          tma_load_2d_pair(st + A_BYTES + B_BYTES + E_BYTES + SF_BYTES, &tmap_sfb, 0,
                           ((prow / 128) * kb128 + 4 * kb) * 2, bar);
          if (two)
            tma_load_2d_pair(st + A_BYTES + B_BYTES + E_BYTES + 2 * SF_BYTES, &tmap_sfb, 0,
                             ((prow / 128 + 1) * kb128 + 4 * kb) * 2, bar);
          ++fills;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: CTA 0 waits until every fill of the pair has landed; CTA 1 until
      // the tensor core has consumed (hence received) its last fill of each slot
      for (int s = 0; s < STAGES; ++s) {
        if (fills > s) {
          const long u = s + (long)STAGES * ((fills - 1 - s) / STAGES);
          const uint32_t par = (uint32_t)((u / STAGES) & 1);
          if (lead) drain_wait(&S.full[s], par);
          else drain_wait(&S.empty[s], par);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer (CTA 0)
    if (lead && elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0u;  // bit b: phase of accumulator buffer b (a register, not an indexed array)
      int buf = 0;
      // Shared-memory descriptors of stage 0 (the same offsets hold the peer's
      // operands); a stage or a K offset only moves the 14-bit start-address
      // field, and all stage addresses stay below 256 KB, so it never carries.
      const uint32_t s0 = smem_u32(smem);
      const uint64_t dA0 = smem_desc(s0, 16, 1024, SWZ_128B);
      const uint64_t dB0 = smem_desc(s0 + A_BYTES, 16, 1024, SWZ_128B);
      const uint64_t dE0 = smem_desc(s0 + A_BYTES + B_BYTES, 16, 128, SWZ_NONE);
      const uint64_t dE2 = smem_desc(s0 + A_BYTES + B_BYTES, BM * 16, 128, SWZ_NONE);  // LBO = chunk stride
      const uint64_t dSFA0 = smem_desc(s0 + A_BYTES + B_BYTES + E_BYTES, 16, 128, SWZ_NONE);
      const uint64_t dSFB0 = dSFA0 + (SF_BYTES >> 4);
      const uint32_t tE = tmem + (NT == 2 ? wide::TM_E : TM_E), tSFA = tmem + (NT == 2 ? wide::TM_SFA : TM_SFA);
      const uint32_t tSFB = tmem + TM_SFB;
      TileWalk walk(S, pair_id, npairs, MT2, E);
      int wpar = 0;  // wide items: accumulator at columns 128 * wpar, alternating per item
      for (int id = pair_id; id < total; id += npairs, walk.advance(MT2)) {
        const Tile t = decode_tile<NT>(S, walk, E);
        const int n_mma = max(16, (t.n_rows + (NT == 2 ? t.n_rows1 : 0) + 15) / 16 * 16);
        const uint32_t idesc = make_idesc<DENSE>((uint32_t)n_mma);
        const uint32_t d_tmem = tmem + TM_ACC + (NT == 2 ? wpar * BN : buf * BN);
        const bool two = NT == 2 && t.n_rows1 > 0;
        mbar_wait_spin(&S.acc_empty[buf], ((acc_phase >> buf) & 1u) ^ 1u, abort, p.d_status);
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          mbar_wait_spin(&S.full[stage], phase, abort, p.d_status);
          tc_fence_after();
          const uint64_t so = (uint64_t)((stage * STAGE_BYTES) >> 4);
          const int nk = min(4, kb128 - 4 * kb);
          if constexpr (NT == 2) {
            // one MMA of N <= 256 per 128 dense K.  The token scales of MMA j take eight
            // TMEM columns: column c holds rows 32c..32c+31 (lane = row % 32, byte =
            // scale), so the second tile's block (rows 128..255) goes to columns 4..7.
            const uint32_t tSFBw = tmem + wide::TM_SFB;
            tc_cp_pair_128x256b(tE, dE2 + so);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_pair_32x128b_warpx4(tSFA + 4 * j, dSFA0 + so + (uint64_t)(j * (512 >> 4)));
              tc_cp_pair_32x128b_warpx4(tSFBw + 8 * j, dSFB0 + so + (uint64_t)(j * (512 >> 4)));
              if (two)
                tc_cp_pair_32x128b_warpx4(tSFBw + 8 * j + 4, dSFB0 + so + (uint64_t)((SF_BYTES + j * 512) >> 4));
              tc_mma_pair_sp_nvf4(d_tmem, dA0 + so + (uint64_t)(j * 2),
                                  dB0 + so + (uint64_t)((j >> 1) * (wide::B_CHUNK >> 4) + (j & 1) * 4), tE + 2 * j,
                                  idesc, tSFA + 4 * j, tSFBw + 8 * j, (kb > 0 || j > 0) ? 1u : 0u);
            }
          } else if constexpr (DENSE) {
            // dense MMAs of 64 dense K: A and B each advance 32 B inside their
            // 128-byte swizzle rows; one scale block per MMA and operand
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (j < nk) {
                tc_cp_pair_32x128b_warpx4(tSFA + 4 * j, dSFA0 + so + (uint64_t)(j * (512 >> 4)));
                tc_cp_pair_32x128b_warpx4(tSFB + 4 * j, dSFB0 + so + (uint64_t)(j * (512 >> 4)));
                tc_mma_pair_nvf4(d_tmem, dA0 + so + (uint64_t)(j * 2), dB0 + so + (uint64_t)(j * 2), idesc,
                                 tSFA + 4 * j, tSFB + 4 * j, (kb > 0 || j > 0) ? 1u : 0u);
              }
            }
          } else if (nk == 4) {
            // metadata of both 256-deep chunks (2 KB apart) in one copy; MMA j
            // reads columns tE + 2j
            tc_cp_pair_128x256b(tE, dE2 + so);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_pair_32x128b_warpx4(tSFA + 4 * j, dSFA0 + so + (uint64_t)(j * (512 >> 4)));
              tc_cp_pair_32x128b_warpx4(tSFB + 4 * j, dSFB0 + so + (uint64_t)(j * (512 >> 4)));
              tc_mma_pair_sp_nvf4(d_tmem, dA0 + so + (uint64_t)(j * 2),
                                  dB0 + so + (uint64_t)((j >> 1) * (B_CHUNK >> 4) + (j & 1) * 4), tE + 2 * j,
                                  idesc, tSFA + 4 * j, tSFB + 4 * j, (kb > 0 || j > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < nk) {
              // metadata of 256 dense K per copy (MMA j reads columns tE + 2j),
              // one scale block per MMA and operand
              if ((j & 1) == 0) tc_cp_pair_128x128b(tE + 2 * j, dE0 + so + (uint64_t)((j >> 1) * (BM * 16 >> 4)));
              tc_cp_pair_32x128b_warpx4(tSFA + 4 * j, dSFA0 + so + (uint64_t)(j * (512 >> 4)));
              tc_cp_pair_32x128b_warpx4(tSFB + 4 * j, dSFB0 + so + (uint64_t)(j * (512 >> 4)));
              // A: +32 B per 128 dense K inside the 128-byte swizzle row; B: 64 B
              // per 128 dense K inside a 256-deep chunk
              tc_mma_pair_sp_nvf4(d_tmem, dA0 + so + (uint64_t)(j * 2),
                                  dB0 + so + (uint64_t)((j >> 1) * (B_CHUNK >> 4) + (j & 1) * 4), tE + 2 * j,
                                  idesc, tSFA + 4 * j, tSFB + 4 * j, (kb > 0 || j > 0) ? 1u : 0u);
            }
          }
          }
          tc_commit_pair_mc(&S.empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        tc_commit_pair_mc(&S.acc_full[buf], 0x3);
        acc_phase ^= 1u << buf;
        if constexpr (NT == 1) buf ^= 1;  // wide items: one barrier pair, alternating columns
        wpar ^= 1;
      }
      // drain: all tensor-core work of the pair complete before TMEM is freed
      tc_commit_pair_mc(&S.done, 0x1);
      drain_wait(&S.done, 0);
    }
    __syncwarp();
  } else {
    // ================================================================ epilogue
    // 16 warps, four per TMEM lane quarter q (rows 32q..32q+31); warp k of a
    // quarter owns token columns [32k, 32k+32).  Lane = accumulator row = output
    // feature.  Each CTA drains its own 128 rows of the pair's accumulator.
    const int ew = warp - 2;            // 0..15
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int kb = ew >> 2;             // column block
    const int c_lo = 32 * kb;           // first column of this warp's block
    uint32_t acc_phase = 0u;  // bit b: phase of accumulator buffer b
    int buf = 0;
    const int I = p.M / 2;
    // accumulator buffer released to CTA 0's MMA warp: a local arrive in CTA 0,
    // a remote one from CTA 1
    const uint32_t acc_empty_lead0 = cluster_map(&S.acc_empty[0], 0), acc_empty_lead1 = cluster_map(&S.acc_empty[1], 0);
    auto release_acc = [&](int b) {
      if (lead) mbar_arrive(&S.acc_empty[b]);
      else mbar_arrive_remote(b ? acc_empty_lead1 : acc_empty_lead0);
    };
    TileWalk walk(S, pair_id, npairs, MT2, E);
    int sb = 0;  // SwiGLU staging buffer of this tile
    [[maybe_unused]] int wpar = 0;  // wide items: accumulator at columns 128 * wpar
    // the next tile is decoded while this one drains (a chain of shared-memory
    // loads that would otherwise stand alone between tiles)
    Tile tn = pair_id < total ? decode_tile<NT>(S, walk, E) : Tile{};
    for (int id = pair_id; id < total; id += npairs) {
      const Tile t = tn;
      auto decode_next = [&]() {
        if (id + npairs < total) {
          walk.advance(MT2);
          tn = decode_tile<NT>(S, walk, E);
        }
      };
      const int mt = 2 * t.mt + (int)rank;  // this CTA's weight tile
      const bool own_tile = mt < MT;          // false: the duplicate of an odd last tile
      const float2 ag = S.ag[t.e];
      const float alpha = ag.x;  // the accumulator's scale (gate rows of gate_up)
      // up rows: the same, or their own global (read before the accumulator wait)
      const float alpha_u = p.exact ? __fmul_rn(__ldg(p.g_act + t.e), __ldg(p.alpha_w + 2 * t.e + 1)) : alpha;
      mbar_wait_poll(&S.acc_full[buf], (acc_phase >> buf) & 1u, abort, p.d_status);
      tc_fence_after();
      const uint32_t tbase = tmem + TM_ACC + buf * BN + ((uint32_t)(32 * q) << 16);
      const bool live = c_lo < t.n_rows;        // any valid token column in the block
      if constexpr (EPI == MOESQ_EPI_SWIGLU_NVFP4) {
        // Tile rows are interleaved (weight repack): in lane quarter q, lanes 16h + j
        // hold the gate rows and lanes 16h + 8 + j the up rows of output
        // o = 16q + 2j + h of this CTA's 64.  A 16x256b load at lane 32q + 16h thus
        // hands thread t the gate and up values of output 16q + 2(t/4) + h for the
        // columns c_lo + 8i + 2(t%4) + b (i < 4, b < 2): no exchange between warps.
        // hv holds h / (alpha * alpha_u) for the raw accumulators g and u: silu(alpha g)
        // = alpha g / (1 + 2^(g * (-alpha log2 e))), so alpha enters the exponent's
        // multiplier and the product alpha * alpha_u enters the amax and the code
        // multiplier below (a few ulp of reassociation, no multiply per element)
        const float ch = __fmul_rn(alpha, alpha_u);
        const float ce = __fmul_rn(alpha, -1.4426950408889634f);
        auto load_h = [&](uint32_t tcol, float (&h_)[2][8]) {
          uint32_t r[16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tmem_ld_16x256b_x4(tcol + ((uint32_t)(16 * h) << 16), r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // columns b = 0, 1 as one packed pair
              const float2 g = make_float2(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]));
              const float2 u = make_float2(__uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
              const float2 hh = __fmul2_rn(sigmoid_scaled2(g, ce), u);
              h_[h][2 * i] = hh.x;
              h_[h][2 * i + 1] = hh.y;
            }
          }
        };
        float hv[2][8];  // [h][v]: v = 2i + b
        [[maybe_unused]] const bool live1 = NT == 2 && c_lo < t.n_rows1;
        if constexpr (NT == 2) {
          // the tile in the shared columns 128-255 (tile 1 at wpar 0, tile 0 at wpar 1)
          // is read first, raw, and the accumulator released; then SiLU, and the other tile
          const uint32_t tsh = tmem + TM_ACC + BN + ((uint32_t)(32 * q) << 16) + c_lo;
          const bool live_sh = wpar ? live : live1;
          uint32_t ra[16], rb[16];
          if (live_sh) {
            tmem_ld_16x256b_x4(tsh, ra);
            tmem_ld_16x256b_x4(tsh + (16u << 16), rb);
            tmem_ld_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(0);
          decode_next();
          auto silu = [&](const uint32_t (&r)[16], float (&h_)[8]) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 g = make_float2(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]));
              const float2 u = make_float2(__uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
              const float2 hh = __fmul2_rn(sigmoid_scaled2(g, ce), u);
              h_[2 * i] = hh.x;
              h_[2 * i + 1] = hh.y;
            }
          };
          if (live_sh) {
            silu(ra, hv[0]);
            silu(rb, hv[1]);
          }
        } else {
          if (live) load_h(tbase + c_lo, hv);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(buf);
          decode_next();
        }
        // amax, scales, codes and stores of one token tile (rows prow_t.., n_t tokens)
        auto finish = [&](const float (&hv)[2][8], int prow_t, int n_t, bool live) {
          if (live) {
            // amax of each column over this warp's 16 outputs: per thread over its two,
            // then over the 8 lanes of equal t%4 (lane bits 2..4) by three halving
            // exchanges; lane t ends with column v = (t >> 2) & 7 of its own t%4
            float m[8];
#pragma unroll
            for (int v = 0; v < 8; ++v) m[v] = fmaxf(fabsf(hv[0][v]), fabsf(hv[1][v]));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const bool hi = lane & 16;
              const float x = __shfl_xor_sync(0xffffffffu, hi ? m[k] : m[k + 4], 16);
              m[k] = fmaxf(hi ? m[k + 4] : m[k], x);
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const bool hi = lane & 8;
              const float x = __shfl_xor_sync(0xffffffffu, hi ? m[k] : m[k + 2], 8);
              m[k] = fmaxf(hi ? m[k + 2] : m[k], x);
            }
            {
              const bool hi = lane & 4;
              const float x = __shfl_xor_sync(0xffffffffu, hi ? m[0] : m[1], 4);
              m[0] = fmaxf(hi ? m[1] : m[0], x);
            }
            // the scale group (32 outputs) spans quarters q and q ^ 1, which use the
            // same lane -> column map: swap the partial amax through shared memory
            float* xa = epi + (kb * 4 + q) * 32;
            xa[lane] = m[0];
            named_bar_sync(2 + (q >> 1) + 2 * kb, 64);
            const float amax = __fmul_rn(fmaxf(m[0], epi[(kb * 4 + (q ^ 1)) * 32 + lane]), fabsf(ch));
            const GroupScale gs = nvfp4_group_scale(amax, ag.y);
            // code multiplier of column (lane >> 2) & 7 for the scaled hv, transposed through
            // shared memory so that each thread reads its 8 columns with two vector loads
            float* xi = epi + 512 + ew * 32;
            xi[(lane & 3) * 8 + ((lane >> 2) & 7)] = __fmul_rn(gs.inv, ch);
            __syncwarp();
            const float4 iv0 = *reinterpret_cast<const float4*>(xi + (lane & 3) * 8);
            const float4 iv1 = *reinterpret_cast<const float4*>(xi + (lane & 3) * 8 + 4);
            const float ivs[8] = {iv0.x, iv0.y, iv0.z, iv0.w, iv1.x, iv1.y, iv1.z, iv1.w};
            const int vc = (lane >> 2) & 7;
            const int rc = 8 * (vc >> 1) + 2 * (lane & 3) + (vc & 1);  // this lane's column (row of the block)
            if ((q & 1) == 0) S.sstg[sb][kb][rc][q >> 1] = (uint8_t)gs.sc;
            // codes: byte 8q + t/4 of each of this thread's 8 token rows (outputs 2(t/4) + {0,1})
            uint8_t* stg = &S.hstg[sb][kb][0][8 * q + (lane >> 2)];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float inv = ivs[v];
              const float2 x = __fmul2_rn(make_float2(hv[0][v], hv[1][v]), make_float2(inv, inv));
              const uint32_t byte = inv == 0.0f ? 0u : e2m1x2(x.x, x.y);
              stg[(8 * (v >> 1) + 2 * (lane & 3) + (v & 1)) * 32] = (uint8_t)byte;
            }
          }
          // the four warps of this column block hold all 64 outputs of its 32 tokens:
          // one TMA store of [32 rows][32 B] codes (rows past the expert's tokens are its
          // own padding, never read as tokens) and 2-byte scale pairs
          fence_proxy_async_smem();
          if (q == 2 && lane == 0) bulk_wait_group_read0();  // the store two tiles back has read its buffer
          named_bar_sync(10 + kb, 128);  // also: both amax slots of every pair are read
          if (live) {
            const int64_t prow0 = (int64_t)prow_t + c_lo;
            if (q == 2 && lane == 0) {
              tma_store_2d(&tmap_y, &S.hstg[sb][kb][0][0], 32 * mt, (int32_t)prow0);
              bulk_commit_group();
            }
            if (q == 3 && lane < n_t - c_lo) {
              const int64_t prow = prow0 + lane;
              const int64_t blk = (prow / 128) * (I / 128) + (64 * mt) / 128;
              *reinterpret_cast<uint16_t*>(p.out_sf + blk * 512 + sf_block_offset((uint32_t)(prow % 128), 2u * (mt & 1))) =
                  *reinterpret_cast<const uint16_t*>(&S.sstg[sb][kb][lane][0]);
            }
          }
          sb ^= 1;
        };
        if constexpr (NT == 2) {
          // the shared-column tile first (its values are in hv), then the other one
          if (wpar) {
            finish(hv, t.prow, t.n_rows, live);
            if (t.n_rows1 > 0) {
              if (live1) load_h(tbase + 2 * BN + c_lo, hv);
              finish(hv, t.prow + BN, t.n_rows1, live1);
            }
          } else {
            if (t.n_rows1 > 0) finish(hv, t.prow + BN, t.n_rows1, live1);
            if (live) load_h(tbase + c_lo, hv);
            finish(hv, t.prow, t.n_rows, live);
          }
          wpar ^= 1;
        } else {
          finish(hv, t.prow, t.n_rows, live);
        }
      } else if constexpr (EPI == MOESQ_EPI_BF16 || EPI == EPI_BF16_COMBINE) {
        // Per 32-token column block kb, its four warps (one per lane quarter q) write
        // [32 tokens][128 outputs] bf16.  The interleaved weight rows put both outputs of
        // a bf16 pair in one thread of a 16x256b TMEM load (down: lanes j and 8 + j of a
        // 16-lane group; gate_up: gate or up of outputs 16q + 2j + {0,1} from the loads
        // at lane 32q and 32q + 16), so each pair is one word and no lanes exchange values.
        // nblk is the same for the block's four warps, so they take the same branch.
        const int64_t s0 = t.s0;
        int nvalid = t.n_rows;
        if (s0 + nvalid > p.S) nvalid = (int)(p.S - s0 > 0 ? p.S - s0 : 0);
        const int nblk = min(32, nvalid - c_lo);  // valid rows of this block (<= 0: none)
        uint32_t r0[16], r1[16];
        if (nblk > 0) {
          tmem_ld_16x256b_x4(tbase + c_lo, r0);
          tmem_ld_16x256b_x4(tbase + (16u << 16) + c_lo, r1);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(buf);
        decode_next();
        const bool gu = p.gate_up;
        const int j = lane >> 2;
        // pair slots of the thread's two words per column
        const int w0 = gu ? 8 * q + j : 16 * (q & 1) + j;
        const int w1 = gu ? w0 : w0 + 8;
        if (EPI == MOESQ_EPI_BF16 && nblk == 32) {
          // a full block: the four warps stage [32 tokens][128 outputs] as two 64-output
          // halves [32 rows][128 B] in the TMA 128-byte swizzle (16-byte chunk c of row r
          // at c ^ (r & 7)) and one lane writes them with two TMA stores.  Words of one
          // staging store land on 8 consecutive pair slots of 4 rows two apart: no bank
          // conflicts.
          uint8_t* stg = reinterpret_cast<uint8_t*>(epi) + kb * 8192;  // [2 halves][32 rows][128 B]
          const bool issuer = q == 2 && lane == 0;
          if (issuer) bulk_wait_group_read0();  // this block's previous stores have read the staging
          named_bar_sync(10 + kb, 128);
          uint8_t* h0 = stg + (gu ? 0 : (q >> 1) * 4096);
          uint8_t* h1 = stg + (gu ? 4096 : (q >> 1) * 4096);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const int i = v >> 1, b = v & 1;
            const int row = 8 * i + 2 * (lane & 3) + b;
            const float a0 = __uint_as_float(r0[4 * i + b]), a1 = __uint_as_float(r0[4 * i + 2 + b]);
            const float c0 = __uint_as_float(r1[4 * i + b]), c1 = __uint_as_float(r1[4 * i + 2 + b]);
            // down: (a0, a1) and (c0, c1) are output pairs; gate_up: (a0, c0) gate, (a1, c1) up
            const float2 w0v = __fmul2_rn(make_float2(a0, gu ? c0 : a1), make_float2(alpha, alpha));
            const float2 w1v = __fmul2_rn(make_float2(gu ? a1 : c0, c1), make_float2(gu ? alpha_u : alpha, gu ? alpha_u : alpha));
            *reinterpret_cast<__nv_bfloat162*>(h0 + row * 128 + (((w0 >> 2) ^ (row & 7)) << 4) + ((w0 & 3) << 2)) =
                __floats2bfloat162_rn(w0v.x, w0v.y);
            *reinterpret_cast<__nv_bfloat162*>(h1 + row * 128 + (((w1 >> 2) ^ (row & 7)) << 4) + ((w1 & 3) << 2)) =
                __floats2bfloat162_rn(w1v.x, w1v.y);
          }
          fence_proxy_async_smem();
          named_bar_sync(10 + kb, 128);  // staging of the block complete
          if (own_tile && issuer) {
            tma_store_2d(&tmap_y, stg, gu ? 64 * mt : BM * mt, (int32_t)(s0 + c_lo));
            tma_store_2d(&tmap_y, stg + 4096, gu ? I + 64 * mt : BM * mt + 64, (int32_t)(s0 + c_lo));
            bulk_commit_group();
          }
        } else if (own_tile && nblk > 0) {
          // a block past the expert's last tokens: each pair word goes straight to global
          // memory; for a fixed (i, b) the eight lanes of equal lane & 3 hold 16
          // consecutive outputs of one token row, so a warp store writes four tokens'
          // 32-byte row segments (whole sectors), with no staging or block barrier
          const int base0 = gu ? 64 * mt : BM * mt + 64 * (q >> 1);
          const int base1 = gu ? I + 64 * mt : base0;
          uint16_t* yb = (uint16_t*)p.out + (s0 + c_lo) * p.M;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const int i = v >> 1, b = v & 1;
            const int row = 8 * i + 2 * (lane & 3) + b;
            const float a0 = __uint_as_float(r0[4 * i + b]), a1 = __uint_as_float(r0[4 * i + 2 + b]);
            const float c0 = __uint_as_float(r1[4 * i + b]), c1 = __uint_as_float(r1[4 * i + 2 + b]);
            const float2 w0v = __fmul2_rn(make_float2(a0, gu ? c0 : a1), make_float2(alpha, alpha));
            const float2 w1v = __fmul2_rn(make_float2(gu ? a1 : c0, c1), make_float2(gu ? alpha_u : alpha, gu ? alpha_u : alpha));
            if (row < nblk) {
              uint16_t* yr = yb + (int64_t)row * p.M;
              *reinterpret_cast<__nv_bfloat162*>(yr + base0 + 2 * w0) = __floats2bfloat162_rn(w0v.x, w0v.y);
              *reinterpret_cast<__nv_bfloat162*>(yr + base1 + 2 * w1) = __floats2bfloat162_rn(w1v.x, w1v.y);
            }
          }
          if constexpr (EPI == EPI_BF16_COMBINE) {
            // Fused weighted combine, deterministic: every (token, 128-output tile) counts
            // its k arrivals, one per slot, each after that slot's y rows are written and
            // fenced; the arrival that completes the count sums the token's k rows of the
            // tile in j order, exactly as the separate combine does (float32, no fused
            // multiply-add, products of the stored bf16 y), and writes the output.  Rows
            // are read at L2 (other SMs wrote them).
            __threadfence();
            named_bar_sync(10 + kb, 128);  // the block's y rows are written and fenced
            const int bt = (ew & 3) * 32 + lane;  // thread of the block
            // per row of the block: the token completed by this arrival, else -1
            volatile int32_t* done = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(epi) + kb * 8192);
            if (bt < 32) {
              int32_t tok_done = -1;
              if (bt < nblk) {
                const int32_t tok = p.slot_token[s0 + c_lo + bt];
                __threadfence();  // release: the block's rows (fenced, then the barrier) before the count
                if (atomicAdd(p.arrivals + (int64_t)tok * MT + mt, 1) == p.k - 1) tok_done = tok;
              }
              done[bt] = tok_done;
              __threadfence();
            }
            named_bar_sync(10 + kb, 128);
            for (int r = ew & 3; r < nblk; r += 4) {
              const int64_t tok = done[r];
              if (tok < 0) continue;
              __threadfence();  // acquire: every arrival's rows before these loads
              // lanes j < k hold slot j and its weight; the rows are loaded eight at a
              // time before they are summed, in j order
              int64_t sl = 0;
              float wl = 0.0f;
              if (lane < p.k) {
                sl = p.token_slot[tok * p.k + lane];
                wl = p.topk_w[tok * p.k + lane];
              }
              float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
              for (int j0 = 0; j0 < p.k; j0 += 8) {
                uint2 uv[8];
                float wv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const int64_t sj = __shfl_sync(0xffffffffu, sl, (j0 + u) & 31);
                  wv[u] = __shfl_sync(0xffffffffu, wl, (j0 + u) & 31);
                  uv[u] = j0 + u < p.k ? __ldcg(reinterpret_cast<const uint2*>((const uint16_t*)p.out + sj * p.M +
                                                                                 BM * mt + 4 * lane))
                                       : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  if (j0 + u < p.k) {
                    const float wj = wv[u];
                    acc[0] = __fadd_rn(acc[0], __fmul_rn(wj, __uint_as_float(uv[u].x << 16)));
                    acc[1] = __fadd_rn(acc[1], __fmul_rn(wj, __uint_as_float(uv[u].x & 0xFFFF0000u)));
                    acc[2] = __fadd_rn(acc[2], __fmul_rn(wj, __uint_as_float(uv[u].y << 16)));
                    acc[3] = __fadd_rn(acc[3], __fmul_rn(wj, __uint_as_float(uv[u].y & 0xFFFF0000u)));
                  }
                }
              }
              const __nv_bfloat162 o0 = __floats2bfloat162_rn(acc[0], acc[1]), o1 = __floats2bfloat162_rn(acc[2], acc[3]);
              uint2 o;
              o.x = *reinterpret_cast<const uint32_t*>(&o0);
              o.y = *reinterpret_cast<const uint32_t*>(&o1);
              *reinterpret_cast<uint2*>(p.comb_out + tok * p.M + BM * mt + 4 * lane) = o;
            }
            named_bar_sync(10 + kb, 128);  // the flags are read before the next tile writes them
          }
        }
      } else {
        // f32: per 16-column half of the block, TMEM (lane = feature) -> swizzled
        // transpose in this warp's shared block -> lanes 0-15 = tokens, one
        // 128-byte row segment each (down: output 16h + 2j + p of the quarter from
        // lane 16h + 8p + j), or two 64-byte segments, gate and up outputs
        // 16q..16q+15 of the tile, from the interleaved lanes (gate_up)
        float* tr = epi + ew * 512;
        const bool gu = p.gate_up;
        const int col0 = BM * mt + 32 * q;
        const int64_t s0 = t.s0;
        int nvalid = t.n_rows;                     // valid columns of the tile
        if (s0 + nvalid > p.S) nvalid = (int)(p.S - s0 > 0 ? p.S - s0 : 0);
        uint32_t acc[32];
        if (c_lo < nvalid) {
          tmem_ld_32x32b_x32(tbase + c_lo, acc);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(buf);
        decode_next();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int cb = c_lo + 16 * h2;
          if (cb < nvalid) {
#pragma unroll
            for (int c = 0; c < 16; ++c) tr[c * 32 + (lane ^ c)] = __uint_as_float(acc[16 * h2 + c]);
            __syncwarp();
            if (own_tile && lane < 16 && lane < nvalid - cb) {
              const int64_t s = s0 + cb + lane;
              float4* y = reinterpret_cast<float4*>((float*)p.out + s * p.M + col0);
              const float* row = tr + lane * 32;
#pragma unroll 1
              for (int u = 0; u < 8; ++u) {
                float v[4];
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                  // output position 4u + z: segment s = pos / 16 at offset o = pos % 16
                  // comes from lane 16 (o & 1) + 8 s + o / 2 in the interleaved rows
                  const int pos = 4 * u + z;
                  const int src = gu ? (((pos & 1) << 4) | ((pos >> 4) << 3) | ((pos & 15) >> 1))
                                     : ((pos & 16) | ((pos & 1) << 3) | ((pos & 15) >> 1));
                  v[z] = __fmul_rn(row[src ^ lane], gu && pos >= 16 ? alpha_u : alpha);
                }
                if (gu) {
                  float* yg = (float*)p.out + s * p.M + (u >= 4 ? I : 0) + 64 * mt + 16 * q + 4 * (u & 3);
                  *reinterpret_cast<float4*>(yg) = make_float4(v[0], v[1], v[2], v[3]);
                } else {
                  y[u] = make_float4(v[0], v[1], v[2], v[3]);
                }
              }
            }
            __syncwarp();
          }
        }
      }
      acc_phase ^= 1u << buf;
      if constexpr (NT == 1) buf ^= 1;
    }
  }

  if constexpr (EPI == MOESQ_EPI_BF16 || EPI == MOESQ_EPI_SWIGLU_NVFP4) {
    if (warp >= 2 && (warp & 3) == 2 && lane == 0) bulk_wait_group0();  // the last stores are complete
  }
  // no CTA of the pair frees TMEM or exits while its peer may still use it
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace sp

// ------------------------------------------------------------------- host ---
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_encodeTiled)ptr;
  });
  return fn;
}

// byte tensor of `rank` dims (innermost first); strides in bytes of dims 1..rank-1
static bool make_tmap_u8(CUtensorMap* m, const void* base, uint32_t rank, const cuuint64_t* dims,
                         const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swz) {
  PFN_encodeTiled enc = get_encode_fn();
  if (!enc) return false;
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool make_tmap_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                           uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_rows};
  return make_tmap_u8(m, base, 2, dims, strides, box, swz);
}

static int device_sms(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
  if (dev_out) *dev_out = dev;
  return major == 10 ? sms : 0;
}

}  // namespace moesq

using namespace moesq;

extern "C" moesq_status moesq_grouped_gemm_workspace_size(const moesq_linear* W, int64_t S,
                                                          size_t* bytes) {
  MOESQ_REQUIRE(W && bytes && S >= 0, MOESQ_ERR_INVALID_ARG);
  *bytes = 0;
  return MOESQ_OK;
}

// Upper bound on the CTA pairs a grouped GEMM launches (0: none), process-wide.
static std::atomic<int> g_pair_limit{0};
// Token tiles per work item of the sparse SwiGLU GEMM: 0 chooses, 1 or 2 forces
// (2 where the shape allows wide items), process-wide.
static std::atomic<int> g_tiles_per_item{0};

// Wide items (two 128-token tiles, one N <= 256 MMA per K step) for the sparse SwiGLU
// gate_up GEMM: K a multiple of 512 (whole stages, so both token chunks of every
// stage are loaded).  Unless forced they are chosen for K >= 4096 and an average of
// 256 or more routed slots per expert, where most items hold two full tiles: with
// K = 2048 an item's main loop is too short to cover the two-tile SwiGLU epilogue,
// which then bounds the GEMM (measured 10 % slower than one-tile items there).
static int tiles_per_item(bool dense, int32_t epilogue, int64_t K, int64_t E, int64_t S) {
  if (dense || epilogue != MOESQ_EPI_SWIGLU_NVFP4 || K % 512 != 0) return 1;
  const int f = g_tiles_per_item.load(std::memory_order_relaxed);
  if (f) return f;
  return K >= 4096 && S >= 256 * E ? 2 : 1;
}

// CTA pairs of a launch: clusters of 2 CTAs, one CTA per SM, as many pairs as the
// device can hold at once (cached per device and kernel), capped by g_pair_limit.
template <bool DENSE>
static moesq_status launch_pairs(int dev, int sms, int32_t epilogue, int* pairs_out, bool wide = false,
                                 bool comb = false) {
  const size_t smem = wide ? sp::smem_bytes_wide() : sp::smem_bytes<DENSE>();
  static int pairs_cache[64][5] = {{0}};
  const int ei = comb ? 4 : wide ? 3 : epilogue - MOESQ_EPI_F32;
  int pairs = dev < 64 ? pairs_cache[dev][ei] : 0;
  if (pairs == 0) {
    const void* fn = comb ? (const void*)sp::k_grouped_gemm_sp<sp::EPI_BF16_COMBINE, false, 1>
                     : wide ? (const void*)sp::k_grouped_gemm_sp<MOESQ_EPI_SWIGLU_NVFP4, false, 2>
                     : epilogue == MOESQ_EPI_F32 ? (const void*)sp::k_grouped_gemm_sp<MOESQ_EPI_F32, DENSE>
                     : epilogue == MOESQ_EPI_BF16 ? (const void*)sp::k_grouped_gemm_sp<MOESQ_EPI_BF16, DENSE>
                                                  : (const void*)sp::k_grouped_gemm_sp<MOESQ_EPI_SWIGLU_NVFP4, DENSE>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOESQ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sms & ~1));
    cfg.blockDim = dim3(sp::THREADS);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      return MOESQ_ERR_CUDA;
    }
    pairs = n < sms / 2 ? n : sms / 2;
    if (dev < 64) pairs_cache[dev][ei] = pairs;
  }
  const int lim = g_pair_limit.load(std::memory_order_relaxed);
  if (lim > 0 && lim < pairs) pairs = lim;
  *pairs_out = pairs;
  return MOESQ_OK;
}

// Both grouped GEMMs: DENSE = false is the paired-4:8 sparse kernel (W->packed are
// the kept bytes, W->meta the sparse metadata); DENSE = true is the comparison
// kernel on decoded weights (W->packed dense codes [E, out, K/2], no metadata, W->sf
// and act_sf in the 16-element scale layout of moesq_sf_expand_block16).
// The weighted combine fused into the down GEMM (moesq_grouped_gemm_down_combine).
struct CombineArgs {
  const int32_t* slot_token;
  const int32_t* token_slot;
  const float* topk_w;
  int64_t T;
  int k;
  uint16_t* out;
  int32_t* arrivals;
};

template <bool DENSE>
static moesq_status grouped_gemm_impl(const moesq_linear* W, const uint8_t* act_codes, const uint8_t* act_sf,
                                      const float* g_act, const int32_t* expert_offsets,
                                      const int32_t* pad_offsets, int64_t S, int64_t P_cap, int32_t epilogue,
                                      const float* g_next, void* out, uint8_t* out_sf, int32_t* d_status,
                                      moesq_stream_t stream, const CombineArgs* comb = nullptr) {
  MOESQ_REQUIRE(W, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(W->packed && (DENSE || W->meta) && W->sf && W->alpha_w, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(act_codes && act_sf && g_act && expert_offsets && pad_offsets && out,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(epilogue >= MOESQ_EPI_F32 && epilogue <= MOESQ_EPI_SWIGLU_NVFP4,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(W->E >= 1 && W->E <= sp::MAX_E && W->out > 0 && W->K > 0 && S >= 0 && P_cap >= 0,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(W->out % 128 == 0 && W->K % 128 == 0 && P_cap % 128 == 0,
                MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(W->out * (int64_t)W->E < (1ll << 31) && W->K < (1 << 20), MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(P_cap >= moesq_padded_rows(S, W->E) && P_cap < (1ll << 31),
                MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(W->kind >= MOESQ_LINEAR_DOWN && W->kind <= MOESQ_LINEAR_GATE_UP_EXACT, MOESQ_ERR_INVALID_ARG);
  const bool gate_up = W->kind != MOESQ_LINEAR_DOWN;
  if (epilogue == MOESQ_EPI_SWIGLU_NVFP4) {
    MOESQ_REQUIRE(gate_up && g_next && out_sf, MOESQ_ERR_INVALID_ARG);
    MOESQ_REQUIRE(W->out % 256 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  }
  if (gate_up) MOESQ_REQUIRE(W->out % 256 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (comb) {
    MOESQ_REQUIRE(!gate_up && epilogue == MOESQ_EPI_BF16, MOESQ_ERR_INVALID_ARG);  // sparse kernel only
    MOESQ_REQUIRE(comb->slot_token && comb->token_slot && comb->topk_w && comb->out && comb->arrivals,
                  MOESQ_ERR_INVALID_ARG);
    MOESQ_REQUIRE(comb->k >= 1 && comb->k <= 32 && comb->T >= 0 && S == comb->T * comb->k, MOESQ_ERR_INVALID_ARG);
    MOESQ_REQUIRE(moesq_aligned16(comb->out), MOESQ_ERR_INVALID_ARG);
  }
  MOESQ_REQUIRE(moesq_aligned16(W->packed) && (DENSE || moesq_aligned16(W->meta)) && moesq_aligned16(W->sf) &&
                    moesq_aligned16(act_codes) && moesq_aligned16(act_sf) && moesq_aligned16(out) &&
                    moesq_aligned16(out_sf),
                MOESQ_ERR_INVALID_ARG);
  if (S == 0) return MOESQ_OK;
  if (comb && cudaMemsetAsync(comb->arrivals, 0, (size_t)comb->T * (size_t)(W->out / 128) * sizeof(int32_t),
                              (cudaStream_t)stream) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  int dev = 0;
  const int sms = device_sms(&dev);
  if (sms < 0) return MOESQ_ERR_CUDA;
  if (sms == 0) return MOESQ_ERR_DEVICE;

  // Weight tile: 128 bytes per row a stage (512 dense K of kept bytes, or 256 dense
  // K of dense codes).  A gate_up tile holds
  // the gate and up rows of 64 outputs in the interleaved order of the weight repack
  // (tile row 32q + 16h + 8s + j = row s*I + 16q + 2j + h of the tile's outputs):
  // a 5-D view (byte, j [stride 2 rows], s [stride I rows], h [stride 1 row],
  // 16-row group [stride 16 rows, expert folded in]) loads it with one copy.  Only
  // coordinates of whole tiles are used, so every byte read lies in the weights.
  CUtensorMap ta, tb, tb16, te, tsfa, tsfb;
  const uint64_t rowA = (uint64_t)(DENSE ? W->K / 2 : W->K / 4);
  // MMAs over K = scale blocks per 128 rows; 256-deep metadata chunks
  const int64_t MT = W->out / 128, kb128 = W->K / sp::Geo<DENSE>::KMMA, nkb256 = (W->K + 255) / 256;
  if (gate_up) {
    const uint64_t I = (uint64_t)(W->out / 2);
    const cuuint64_t dims[5] = {rowA, 8, 2, 2, (uint64_t)(W->E * W->out / 16)};
    const cuuint64_t strides[4] = {2 * rowA, I * rowA, rowA, 16 * rowA};
    const cuuint32_t box[5] = {128, 8, 2, 2, 4};
    if (!make_tmap_u8(&ta, W->packed, 5, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return MOESQ_ERR_CUDA;
  } else {
    // down: tile row 16g + 8p + j = row 16g + 2j + p of the tile: (byte, j [stride 2
    // rows], p [stride 1 row], 16-row group [stride 16 rows, expert folded in])
    const cuuint64_t dims[4] = {rowA, 8, 2, (uint64_t)(W->E * W->out / 16)};
    const cuuint64_t strides[3] = {2 * rowA, rowA, 16 * rowA};
    const cuuint32_t box[4] = {128, 8, 2, 8};
    if (!make_tmap_u8(&ta, W->packed, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return MOESQ_ERR_CUDA;
  }
  // token codes: a CTA stages 64 (or, for tiles of <= 32 tokens, 16) rows
  if (!make_tmap_rows(&tb, act_codes, (uint64_t)(W->K / 2), (uint64_t)P_cap, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_rows(&tb16, act_codes, (uint64_t)(W->K / 2), (uint64_t)P_cap, 128, 16,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return MOESQ_ERR_CUDA;
  // the same token codes as (128-byte chunk row, row, 256-deep chunk): both 64-row chunks
  // of a 512-deep stage in one box; valid when K % 256 == 0 (else the 2-D boxes are used)
  CUtensorMap tb3 = tb;
  if (!DENSE && W->K % 256 == 0) {
    const cuuint64_t dims[3] = {128, (uint64_t)P_cap, (uint64_t)(W->K / 256)};
    const cuuint64_t strides[2] = {(uint64_t)(W->K / 2), 128};
    const cuuint32_t box64[3] = {128, 64, 2};
    if (!make_tmap_u8(&tb3, act_codes, 3, dims, strides, box64, CU_TENSOR_MAP_SWIZZLE_128B)) return MOESQ_ERR_CUDA;
  }
  // wide items: a CTA's 128 rows of both chunks in one box (32 KB)
  const bool wide = tiles_per_item(DENSE, epilogue, W->K, W->E, S) == 2;
  if (wide) {
    const cuuint64_t dims[3] = {128, (uint64_t)P_cap, (uint64_t)(W->K / 256)};
    const cuuint64_t strides[2] = {(uint64_t)(W->K / 2), 128};
    const cuuint32_t box128[3] = {128, 128, 2};
    if (!make_tmap_u8(&tb3, act_codes, 3, dims, strides, box128, CU_TENSOR_MAP_SWIZZLE_128B)) return MOESQ_ERR_CUDA;
  }
  // metadata and scale blocks seen as 256-byte rows (no swizzle: contiguous copies)
  te = ta;  // unused by the dense kernel
  if ((!DENSE && !make_tmap_rows(&te, W->meta, 256, (uint64_t)(W->E * MT * nkb256 * 8), 256, 16,
                                 CU_TENSOR_MAP_SWIZZLE_NONE)) ||
      !make_tmap_rows(&tsfa, W->sf, 256, (uint64_t)(W->E * MT * kb128 * 2), 256, 8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_rows(&tsfb, act_sf, 256, (uint64_t)(P_cap / 128 * kb128 * 2), 256, 8,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return MOESQ_ERR_CUDA;

  // bf16 output [S rows x out columns]: 64-column x 128-row boxes, 128-byte swizzle
  CUtensorMap ty = ta;
  if (epilogue == MOESQ_EPI_SWIGLU_NVFP4) {
    // requantised codes [P_cap rows x I/2 bytes], 32-byte x 32-row boxes, no swizzle
    const cuuint64_t dims[2] = {(uint64_t)(W->out / 4), (uint64_t)P_cap};
    const cuuint64_t strides[1] = {(uint64_t)(W->out / 4)};
    const cuuint32_t box[2] = {32, 32};
    if (!make_tmap_u8(&ty, out, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return MOESQ_ERR_CUDA;
  }
  if (epilogue == MOESQ_EPI_BF16) {
    PFN_encodeTiled enc = get_encode_fn();
    const cuuint64_t dims[2] = {(uint64_t)W->out, (uint64_t)S};
    const cuuint64_t strides[1] = {(uint64_t)W->out * 2};
    const cuuint32_t box[2] = {64, 32}, estr[2] = {1, 1};
    if (!enc || enc(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MOESQ_ERR_CUDA;
  }

  const size_t smem = wide ? sp::smem_bytes_wide() : sp::smem_bytes<DENSE>();
  int pairs = 0;
  const moesq_status pst = launch_pairs<DENSE>(dev, sms, epilogue, &pairs, wide, comb != nullptr);
  if (pst != MOESQ_OK) return pst;
  sp::Params prm;
  prm.meta = W->meta;
  prm.sfw = W->sf;
  prm.alpha_w = W->alpha_w;
  prm.act_sf = act_sf;
  prm.g_act = g_act;
  prm.expert_offsets = expert_offsets;
  prm.pad_offsets = pad_offsets;
  prm.g_next = g_next;
  prm.out = out;
  prm.out_sf = out_sf;
  prm.d_status = d_status;
  prm.E = W->E;
  prm.M = (int)W->out;
  prm.K = (int)W->K;
  prm.epi = epilogue;
  prm.gate_up = gate_up ? 1 : 0;
  prm.exact = W->kind == MOESQ_LINEAR_GATE_UP_EXACT ? 1 : 0;
  prm.S = S;
  prm.P_cap = P_cap;
  prm.slot_token = comb ? comb->slot_token : nullptr;
  prm.token_slot = comb ? comb->token_slot : nullptr;
  prm.topk_w = comb ? comb->topk_w : nullptr;
  prm.arrivals = comb ? comb->arrivals : nullptr;
  prm.comb_out = comb ? comb->out : nullptr;
  prm.k = comb ? comb->k : 0;
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid((unsigned)(2 * pairs));
  cudaError_t err;
  switch (epilogue) {
    case MOESQ_EPI_F32:
      err = moesq_launch(sp::k_grouped_gemm_sp<MOESQ_EPI_F32, DENSE>, grid, dim3(sp::THREADS), smem, st, ta, tb,
                         tb16, te, tsfa, tsfb, ty, tb3, prm);
      break;
    case MOESQ_EPI_BF16:
      if (comb)
        err = moesq_launch(sp::k_grouped_gemm_sp<sp::EPI_BF16_COMBINE, false, 1>, grid, dim3(sp::THREADS), smem, st,
                           ta, tb, tb16, te, tsfa, tsfb, ty, tb3, prm);
      else
        err = moesq_launch(sp::k_grouped_gemm_sp<MOESQ_EPI_BF16, DENSE>, grid, dim3(sp::THREADS), smem, st, ta, tb,
                           tb16, te, tsfa, tsfb, ty, tb3, prm);
      break;
    default:
      if (wide)
        err = moesq_launch(sp::k_grouped_gemm_sp<MOESQ_EPI_SWIGLU_NVFP4, false, 2>, grid, dim3(sp::THREADS), smem,
                           st, ta, tb, tb16, te, tsfa, tsfb, ty, tb3, prm);
      else
        err = moesq_launch(sp::k_grouped_gemm_sp<MOESQ_EPI_SWIGLU_NVFP4, DENSE>, grid, dim3(sp::THREADS), smem, st,
                           ta, tb, tb16, te, tsfa, tsfb, ty, tb3, prm);
  }
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    return MOESQ_ERR_CUDA;
  }
  return MOESQ_OK;
}

extern "C" moesq_status moesq_grouped_gemm(const moesq_linear* W, const uint8_t* act_codes,
                                           const uint8_t* act_sf, const float* g_act,
                                           const int32_t* expert_offsets,
                                           const int32_t* pad_offsets, int64_t S, int64_t P_cap,
                                           int32_t epilogue, const float* g_next, void* out,
                                           uint8_t* out_sf, void* ws, size_t ws_bytes,
                                           int32_t* d_status, moesq_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  return grouped_gemm_impl<false>(W, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap, epilogue,
                                  g_next, out, out_sf, d_status, stream);
}

extern "C" moesq_status moesq_grouped_gemm_down_combine(
    const moesq_linear* W, const uint8_t* act_codes, const uint8_t* act_sf, const float* g_act,
    const int32_t* expert_offsets, const int32_t* pad_offsets, int64_t S, int64_t P_cap, const int32_t* slot_token,
    const int32_t* token_slot, const float* topk_w, int64_t T, int32_t k, uint16_t* y, uint16_t* out,
    int32_t* arrivals, int32_t* d_status, moesq_stream_t stream) {
  const CombineArgs c{slot_token, token_slot, topk_w, T, k, out, arrivals};
  return grouped_gemm_impl<false>(W, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap, MOESQ_EPI_BF16,
                                  nullptr, y, nullptr, d_status, stream, &c);
}

extern "C" moesq_status moesq_grouped_gemm_dense(const moesq_linear* W, const uint8_t* act_codes,
                                                 const uint8_t* act_sf, const float* g_act,
                                                 const int32_t* expert_offsets, const int32_t* pad_offsets,
                                                 int64_t S, int64_t P_cap, int32_t epilogue,
                                                 const float* g_next, void* out, uint8_t* out_sf,
                                                 int32_t* d_status, moesq_stream_t stream) {
  return grouped_gemm_impl<true>(W, act_codes, act_sf, g_act, expert_offsets, pad_offsets, S, P_cap, epilogue,
                                 g_next, out, out_sf, d_status, stream);
}

extern "C" moesq_status moesq_set_gemm_pair_limit(int32_t max_pairs) {
  MOESQ_REQUIRE(max_pairs >= 0, MOESQ_ERR_INVALID_ARG);
  g_pair_limit.store(max_pairs, std::memory_order_relaxed);
  return MOESQ_OK;
}

extern "C" moesq_status moesq_gemm_launch_pairs(int32_t dense, int32_t epilogue, int32_t* pairs) {
  MOESQ_REQUIRE(pairs && epilogue >= MOESQ_EPI_F32 && epilogue <= MOESQ_EPI_SWIGLU_NVFP4, MOESQ_ERR_INVALID_ARG);
  int dev = 0;
  const int sms = device_sms(&dev);
  if (sms < 0) return MOESQ_ERR_CUDA;
  if (sms == 0) return MOESQ_ERR_DEVICE;
  int n = 0;
  const moesq_status st =
      dense ? launch_pairs<true>(dev, sms, epilogue, &n) : launch_pairs<false>(dev, sms, epilogue, &n);
  if (st == MOESQ_OK) *pairs = n;
  return st;
}

extern "C" moesq_status moesq_set_gemm_tiles_per_item(int32_t tiles) {
  MOESQ_REQUIRE(tiles >= 0 && tiles <= 2, MOESQ_ERR_INVALID_ARG);
  g_tiles_per_item.store(tiles, std::memory_order_relaxed);
  return MOESQ_OK;
}

extern "C" moesq_status moesq_gemm_tiles_per_item(int32_t dense, int32_t epilogue, int64_t K, int64_t E, int64_t S,
                                                  int32_t* tiles) {
  MOESQ_REQUIRE(tiles && epilogue >= MOESQ_EPI_F32 && epilogue <= MOESQ_EPI_SWIGLU_NVFP4 && K > 0 && E > 0 && S >= 0,
                MOESQ_ERR_INVALID_ARG);
  *tiles = tiles_per_item(dense != 0, epilogue, K, E, S);
  return MOESQ_OK;
}
