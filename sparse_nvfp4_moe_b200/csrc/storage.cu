// Pair-bitmask storage codecs, weight export and load-time repack.
//
// Storage ("Sparse storage layout (paired48_sparse, pair-bitmask v1)",
// Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card): packed NVFP4 keeps two adjacent
// K elements per byte, so one kept pair is one byte; every 4-byte chunk keeps 2
// bytes.  weight_sparse_packed [out, K/4] = kept bytes in K order;
// weight_sparse_mask [out, K/16] = 4 bits per chunk, bit i = byte i kept, low
// nibble = lower-K chunk.  All kernels here are HBM-bound byte shuffles: one
// thread per mask byte (16 dense K), 4-/8-byte vector accesses, grids sized to
// a few waves of the 148 SMs.
#include "common.cuh"

namespace moesq {


static inline int grid_for(int64_t n, int block) {
  int64_t g = (n + block - 1) / block;
  const int64_t cap = 148 * 32;
  return (int)(g < cap ? (g > 0 ? g : 1) : cap);
}

// kept byte positions of a legal mask nibble (exactly two bits set): lowest and
// highest set bit; legality is popc == 2
__device__ __forceinline__ bool nib_legal(uint32_t nib) { return __popc(nib) == 2; }
__device__ __forceinline__ uint32_t nib_lo(uint32_t nib) { return __ffs(nib) - 1; }
__device__ __forceinline__ uint32_t nib_hi(uint32_t nib) { return 31 - __clz(nib); }

// one mask byte (two chunks) + its 4 packed bytes -> 8 dense bytes
__device__ __forceinline__ uint2 decode_byte(uint32_t m, uint32_t pk, bool& bad) {
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t nib = (m >> (4 * h)) & 0xF;
    if (!nib_legal(nib)) {
      bad = true;
      out[h] = 0u;
      continue;
    }
    const uint32_t b0 = (pk >> (16 * h)) & 0xFF, b1 = (pk >> (16 * h + 8)) & 0xFF;
    out[h] = (b0 << (8 * nib_lo(nib))) | (b1 << (8 * nib_hi(nib)));
  }
  return make_uint2(out[0], out[1]);
}

// ------------------------------------------------------------------ decode --
// thread per 16 mask bytes: 16 B mask + 64 B packed in -> 128 B dense out (16-byte
// vector accesses); a tail of < 16 mask bytes one byte per thread
__global__ void k_decode(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ mask,
                         uint8_t* __restrict__ dense, int64_t nbytes_mask, int32_t* d_status) {
  bool bad = false;
  const int64_t n16 = nbytes_mask / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += stride) {
    const uint4 mv = reinterpret_cast<const uint4*>(mask)[i];
    const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
    const uint4* pk = reinterpret_cast<const uint4*>(packed) + 4 * i;
    uint4* out = reinterpret_cast<uint4*>(dense) + 8 * i;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 pv = pk[q];  // packed bytes of mask word q (4 mask bytes)
      const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
      uint2 d[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) d[j] = decode_byte((mw[q] >> (8 * j)) & 0xFF, pw[j], bad);
      out[2 * q] = make_uint4(d[0].x, d[0].y, d[1].x, d[1].y);
      out[2 * q + 1] = make_uint4(d[2].x, d[2].y, d[3].x, d[3].y);
    }
  }
  for (int64_t i = 16 * n16 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes_mask; i += stride) {
    const uint2 d = decode_byte(mask[i], *reinterpret_cast<const uint32_t*>(packed + 4 * i), bad);
    *reinterpret_cast<uint2*>(dense + 8 * i) = d;
  }
  if (bad) flag(d_status, MOESQ_DFLAG_BAD_SPARSITY);
}

// ------------------------------------------------------------------ encode --
// 8 dense bytes (two chunks) -> 4 packed bytes + 1 mask byte
// returns (packed word, mask byte)
__device__ __forceinline__ uint2 encode_byte(uint2 d, uint32_t hm, bool use_hint, bool& bad) {
  uint32_t mk = 0, pk = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t w = h ? d.y : d.x;
    uint32_t nz = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) nz |= (((w >> (8 * b)) & 0xFF) != 0) << b;
    uint32_t nib;
    if (use_hint) {
      nib = (hm >> (4 * h)) & 0xF;
      if (!nib_legal(nib) || (nz & ~nib)) bad = true;
    } else {
      nib = nz;
      if (__popc(nib) > 2) bad = true;
      // fill up to 2 kept bytes with the lowest-index zero bytes
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (__popc(nib) < 2 && !((nib >> b) & 1)) nib |= 1u << b;
    }
    if (!nib_legal(nib)) nib = 3;  // only reachable when flagged: keep memory-safe output
    const uint32_t b0 = (w >> (8 * nib_lo(nib))) & 0xFF, b1 = (w >> (8 * nib_hi(nib))) & 0xFF;
    pk |= (b0 | (b1 << 8)) << (16 * h);
    mk |= nib << (4 * h);
  }
  return make_uint2(pk, mk);
}

// thread per 16 mask bytes: 128 B dense (+ 16 B hint) in -> 64 B packed + 16 B mask out
__global__ void k_encode(const uint8_t* __restrict__ dense, const uint8_t* __restrict__ hint,
                         uint8_t* __restrict__ packed, uint8_t* __restrict__ mask,
                         int64_t nbytes_mask, int32_t* d_status) {
  bool bad = false;
  const bool use_hint = hint != nullptr;
  const int64_t n16 = nbytes_mask / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += stride) {
    uint32_t hw[4] = {0u, 0u, 0u, 0u};
    if (use_hint) {
      const uint4 hv = reinterpret_cast<const uint4*>(hint)[i];
      hw[0] = hv.x, hw[1] = hv.y, hw[2] = hv.z, hw[3] = hv.w;
    }
    const uint4* dv = reinterpret_cast<const uint4*>(dense) + 8 * i;
    uint4* pk_out = reinterpret_cast<uint4*>(packed) + 4 * i;
    uint32_t mw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 a = dv[2 * q], c = dv[2 * q + 1];
      const uint2 d[4] = {make_uint2(a.x, a.y), make_uint2(a.z, a.w), make_uint2(c.x, c.y), make_uint2(c.z, c.w)};
      uint2 r[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) r[j] = encode_byte(d[j], (hw[q] >> (8 * j)) & 0xFF, use_hint, bad);
      mw[q] = r[0].y | (r[1].y << 8) | (r[2].y << 16) | (r[3].y << 24);
      pk_out[q] = make_uint4(r[0].x, r[1].x, r[2].x, r[3].x);
    }
    reinterpret_cast<uint4*>(mask)[i] = make_uint4(mw[0], mw[1], mw[2], mw[3]);
  }
  for (int64_t i = 16 * n16 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes_mask; i += stride) {
    const uint2 r = encode_byte(*reinterpret_cast<const uint2*>(dense + 8 * i), use_hint ? hint[i] : 0u, use_hint,
                                bad);
    *reinterpret_cast<uint32_t*>(packed + 4 * i) = r.x;
    mask[i] = (uint8_t)r.y;
  }
  if (bad) flag(d_status, MOESQ_DFLAG_BAD_SPARSITY);
}

// ------------------------------------------------------------ weight export --
// pass 1: paired-4:8 prune (mask) and per-segment amax of the kept values.
// thread per 32-element group (4 chunks): 64 bytes of bf16 in, 2 mask bytes out.
__device__ __forceinline__ void load_group_bf16(const uint16_t* p, float (&v)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = q[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16_bits_to_float(w[j] & 0xFFFF);
      v[8 * i + 2 * j + 1] = bf16_bits_to_float(w[j] >> 16);
    }
  }
}

// keep-bits of the 4 pairs of one chunk: the 2 largest a*a+b*b, ties to the lower pair
__device__ __forceinline__ uint32_t prune_chunk(const float* c) {
  float sc[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) sc[p] = __fadd_rn(__fmul_rn(c[2 * p], c[2 * p]), __fmul_rn(c[2 * p + 1], c[2 * p + 1]));
  uint32_t nib = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    int rank = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) rank += (sc[q] > sc[p]) || (sc[q] == sc[p] && q < p);
    if (rank < 2) nib |= 1u << p;
  }
  return nib;
}

__global__ void k_prune_amax(const uint16_t* __restrict__ w, int64_t E, int64_t out, int64_t K,
                             int32_t n_seg, uint8_t* __restrict__ mask,
                             uint32_t* __restrict__ seg_amax) {
  const int64_t groups_per_row = K / 32;
  const int64_t n = E * out * groups_per_row;
  const int64_t seg_rows = out / n_seg;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / groups_per_row;  // global row e*out + m
    float v[32];
    load_group_bf16(w + 32 * i, v);
    uint32_t m16 = 0;
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t nib = prune_chunk(v + 8 * c);
      m16 |= nib << (4 * c);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if ((nib >> p) & 1) amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * p]), fabsf(v[8 * c + 2 * p + 1])));
    }
    *reinterpret_cast<uint16_t*>(mask + 2 * i) = (uint16_t)m16;
    // one atomic per warp when the whole warp is in one segment
    // (nonnegative floats order as their bit patterns)
    const int64_t e = row / out, seg = (row % out) / seg_rows;
    const uint32_t key = (uint32_t)(e * n_seg + seg);
    const unsigned act = __activemask();
    const int leader = __ffs(act) - 1;
    const uint32_t key0 = __shfl_sync(act, key, leader);
    if (__all_sync(act, key == key0)) {
      const uint32_t mx = __reduce_max_sync(act, __float_as_uint(amax));
      if ((int)(threadIdx.x & 31) == leader) atomicMax(seg_amax + key, mx);
    } else {
      atomicMax(seg_amax + key, __float_as_uint(amax));
    }
  }
}

// pass 2: quantise the kept values and write the packed bytes and block scales.
__global__ void k_quant_encode(const uint16_t* __restrict__ w, int64_t E, int64_t out, int64_t K,
                               int32_t n_seg, const uint8_t* __restrict__ mask,
                               const uint32_t* __restrict__ seg_amax, uint8_t* __restrict__ packed,
                               uint8_t* __restrict__ scale, float* __restrict__ g_w) {
  const int64_t groups_per_row = K / 32;
  const int64_t n = E * out * groups_per_row;
  const int64_t seg_rows = out / n_seg;
  const int64_t tid0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (tid0 < E * n_seg) g_w[tid0] = __fdiv_rn(__uint_as_float(seg_amax[tid0]), 2688.0f);
  for (int64_t i = tid0; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / groups_per_row;
    const int64_t e = row / out, seg = (row % out) / seg_rows;
    const float g = __fdiv_rn(__uint_as_float(seg_amax[e * n_seg + seg]), 2688.0f);
    float v[32];
    load_group_bf16(w + 32 * i, v);
    const uint32_t m16 = *reinterpret_cast<const uint16_t*>(mask + 2 * i);
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if ((m16 >> (4 * c + p)) & 1)
          amax = fmaxf(amax, fmaxf(fabsf(v[8 * c + 2 * p]), fabsf(v[8 * c + 2 * p + 1])));
    const GroupScale gs = nvfp4_group_scale(amax, g);
    // the 16 kept values in K order (2 pairs per chunk) -> 8 kept bytes
    float kept[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t nib = (m16 >> (4 * c)) & 0xF;
      int k = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        if ((nib >> p) & 1) {
          if (k < 2) {
            kept[4 * c + 2 * k] = v[8 * c + 2 * p];
            kept[4 * c + 2 * k + 1] = v[8 * c + 2 * p + 1];
          }
          ++k;
        }
      }
    }
    uint32_t outw[2] = {nvfp4_word(kept, gs.inv), nvfp4_word(kept + 8, gs.inv)};
    *reinterpret_cast<uint2*>(packed + 8 * i) = make_uint2(outw[0], outw[1]);
    scale[i] = (uint8_t)gs.sc;
  }
}

// ------------------------------------------------------------------- repack --
// metadata: thread per (expert, tile, kb256, tile row): 16 mask bytes -> 16 metadata
// bytes.  The metadata nibble of a chunk is i0 | i1 << 2, its kept pair indices
// (lowest and highest set bit of the mask nibble).
// Source row of tile row r.  down: row r = 16g + 8p + j of tile t is row
// 128t + 16g + 2j + p, so that one TMEM load of 16 lanes gives a thread two
// neighbouring outputs.  gate_up: row r = 32q + 16h + 8s + j of tile t is output
// f = 64t + 16q + 2j + h of the gate (s = 0) or up (s = 1) rows, so that the same
// load gives a thread the gate and up values of output f.
__device__ __forceinline__ int64_t tile_src_row(int64_t tile, int64_t r, int64_t out, bool gate_up) {
  if (!gate_up) return 128 * tile + (r & ~15) + 2 * (r & 7) + ((r >> 3) & 1);
  const int64_t I = out / 2;
  const int64_t q = r >> 5, h = (r >> 4) & 1, s = (r >> 3) & 1, j = r & 7;
  return s * I + 64 * tile + 16 * q + 2 * j + h;
}

__device__ __forceinline__ uint32_t meta_of_mask_word(uint32_t w, bool& bad) {
  uint32_t o = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t nib = (w >> (4 * c)) & 0xF;
    const bool ok = nib_legal(nib);
    if (!ok) bad = true;
    o |= (ok ? (nib_lo(nib) | (nib_hi(nib) << 2)) : 0u) << (4 * c);
  }
  return o;
}

__global__ void k_repack_meta(const uint8_t* __restrict__ mask, int64_t E, int64_t out, int64_t K,
                              bool gate_up, uint8_t* __restrict__ meta, int32_t* d_status) {
  const int64_t tiles = out / 128, nkb = (K + 255) / 256, mbytes_row = K / 16;
  const int64_t n = E * tiles * nkb * 128;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i % 128;
    const int64_t kb = (i / 128) % nkb;
    const int64_t t = (i / (128 * nkb)) % tiles;
    const int64_t e = i / (128 * nkb * tiles);
    const int64_t src = e * out + tile_src_row(t, r, out, gate_up);
    const uint8_t* m = mask + src * mbytes_row + kb * 16;
    // rows are K/16 bytes with K % 128 == 0: 8-byte aligned; the last 128 dense K
    // of a row with K % 256 == 128 has 8 mask bytes and zero metadata after them
    const bool full = mbytes_row - kb * 16 >= 16;
    const uint2 m0 = *reinterpret_cast<const uint2*>(m);
    const uint2 m1 = full ? *reinterpret_cast<const uint2*>(m + 8) : make_uint2(0u, 0u);
    uint4 o;
    o.x = meta_of_mask_word(m0.x, bad);
    o.y = meta_of_mask_word(m0.y, bad);
    o.z = full ? meta_of_mask_word(m1.x, bad) : 0u;
    o.w = full ? meta_of_mask_word(m1.y, bad) : 0u;
    // block (e, t, kb) is 2048 bytes, row r at 16 r
    *reinterpret_cast<uint4*>(meta + (((e * tiles + t) * nkb + kb) * 128 + r) * 16) = o;
  }
  if (bad) flag(d_status, MOESQ_DFLAG_BAD_SPARSITY);
}

// scale factors: thread per (expert, tile, kb128, lane l of the block): the 4 scale
// bytes of tile rows l, l+32, l+64, l+96 form the 16 bytes at 16 l of the
// 512-byte block (row r, scale j at (r%32)*16 + (r/32)*4 + j), so a warp writes
// one whole block; up rows of a split gate_up get the up/gate global ratio folded
__global__ void k_repack_sf(const uint8_t* __restrict__ scale, const float* __restrict__ g_w,
                            int64_t E, int64_t out, int64_t K, int32_t kind,
                            uint8_t* __restrict__ sf, float* __restrict__ alpha_w) {
  const bool gate_up = kind != MOESQ_LINEAR_DOWN;
  const bool split = kind == MOESQ_LINEAR_GATE_UP_SPLIT;   // fold the up/gate ratio
  const bool exact = kind == MOESQ_LINEAR_GATE_UP_EXACT;   // keep both globals
  const int64_t tiles = out / 128, nkb = K / 128, sbytes_row = K / 32;
  const int64_t n = E * tiles * nkb * 32;
  const int64_t tid0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (tid0 < E) {
    if (exact) {
      alpha_w[2 * tid0] = g_w[2 * tid0];
      alpha_w[2 * tid0 + 1] = g_w[2 * tid0 + 1];
    } else {
      alpha_w[tid0] = split ? g_w[2 * tid0] : g_w[tid0];
    }
  }
  for (int64_t i = tid0; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t l = i % 32;
    const int64_t kb = (i / 32) % nkb;
    const int64_t t = (i / (32 * nkb)) % tiles;
    const int64_t e = i / (32 * nkb * tiles);
    uint32_t s4[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t srow = tile_src_row(t, l + 32 * c, out, gate_up);
      uint32_t v = *reinterpret_cast<const uint32_t*>(scale + (e * out + srow) * sbytes_row + 4 * kb);
      if (split && srow >= out / 2) {
        const float ratio = __fdiv_rn(g_w[2 * e + 1], g_w[2 * e]);
        uint32_t f = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          f |= e4m3_code(__fmul_rn(e4m3_value((v >> (8 * j)) & 0xFF), ratio)) << (8 * j);
        v = f;
      }
      s4[c] = v;
    }
    *reinterpret_cast<uint4*>(sf + ((e * tiles + t) * nkb + kb) * 512 + 16 * l) =
        make_uint4(s4[0], s4[1], s4[2], s4[3]);
  }
}

}  // namespace moesq

using namespace moesq;

extern "C" moesq_status moesq_decode(const uint8_t* packed, const uint8_t* mask, uint8_t* dense,
                                     int64_t rows, int64_t K, int32_t* d_status,
                                     moesq_stream_t stream) {
  MOESQ_REQUIRE(packed && mask && dense, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(rows >= 0 && K >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(packed) && moesq_aligned16(mask) && moesq_aligned16(dense),
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 64 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  const int64_t n = rows * (K / 16);
  if (n == 0) return MOESQ_OK;
  k_decode<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(packed, mask, dense, n, d_status);
  MOESQ_CHECK_LAUNCH();
  return MOESQ_OK;
}

extern "C" moesq_status moesq_encode(const uint8_t* dense, const uint8_t* mask_hint,
                                     uint8_t* packed, uint8_t* mask, int64_t rows, int64_t K,
                                     int32_t* d_status, moesq_stream_t stream) {
  MOESQ_REQUIRE(dense && packed && mask, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(rows >= 0 && K >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(dense) && moesq_aligned16(packed) && moesq_aligned16(mask) &&
                    moesq_aligned16(mask_hint),
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 64 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  const int64_t n = rows * (K / 16);
  if (n == 0) return MOESQ_OK;
  k_encode<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(dense, mask_hint, packed, mask, n,
                                                               d_status);
  MOESQ_CHECK_LAUNCH();
  return MOESQ_OK;
}

extern "C" moesq_status moesq_quant_weight_workspace_size(int64_t E, int32_t n_seg,
                                                          size_t* bytes) {
  MOESQ_REQUIRE(bytes && E >= 0 && (n_seg == 1 || n_seg == 2), MOESQ_ERR_INVALID_ARG);
  *bytes = (size_t)(E * n_seg) * sizeof(uint32_t);
  return MOESQ_OK;
}

extern "C" moesq_status moesq_quant_weight(const uint16_t* w, int64_t E, int64_t out, int64_t K,
                                           int32_t n_seg, uint8_t* packed, uint8_t* mask,
                                           uint8_t* scale, float* g_w, void* ws, size_t ws_bytes,
                                           moesq_stream_t stream) {
  MOESQ_REQUIRE(w && packed && mask && scale && g_w, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(E >= 0 && out >= 0 && K >= 0 && (n_seg == 1 || n_seg == 2), MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(w) && moesq_aligned16(packed) && moesq_aligned16(mask) &&
                    moesq_aligned16(scale),
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(K % 64 == 0 && out % n_seg == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  size_t need = 0;
  moesq_quant_weight_workspace_size(E, n_seg, &need);
  MOESQ_REQUIRE(ws && ws_bytes >= need, MOESQ_ERR_WORKSPACE);
  if (E * out == 0) return MOESQ_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, need, s) != cudaSuccess) return MOESQ_ERR_CUDA;
  const int64_t n = E * out * (K / 32);
  k_prune_amax<<<grid_for(n, 128), 128, 0, s>>>(w, E, out, K, n_seg, mask, (uint32_t*)ws);
  MOESQ_CHECK_LAUNCH();
  k_quant_encode<<<grid_for(n, 128), 128, 0, s>>>(w, E, out, K, n_seg, mask, (const uint32_t*)ws,
                                                  packed, scale, g_w);
  MOESQ_CHECK_LAUNCH();
  return MOESQ_OK;
}

extern "C" moesq_status moesq_repack_sizes(int64_t out, int64_t K, size_t* meta_bytes,
                                           size_t* sf_bytes) {
  MOESQ_REQUIRE(meta_bytes && sf_bytes && out >= 0 && K >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(out % 128 == 0 && K % 128 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  *meta_bytes = (size_t)(out / 128) * (size_t)((K + 255) / 256) * 2048;
  *sf_bytes = (size_t)(out / 128) * (size_t)(K / 128) * 512;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_repack_meta(const uint8_t* mask, const uint8_t* scale,
                                          const float* g_w, int64_t E, int64_t out, int64_t K,
                                          int32_t kind, uint8_t* meta, uint8_t* sf,
                                          float* alpha_w, int32_t* d_status,
                                          moesq_stream_t stream) {
  MOESQ_REQUIRE(mask && scale && g_w && meta && sf && alpha_w, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(E >= 0 && out >= 0 && K >= 0, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(kind >= MOESQ_LINEAR_DOWN && kind <= MOESQ_LINEAR_GATE_UP_EXACT,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(moesq_aligned16(mask) && moesq_aligned16(scale) && moesq_aligned16(meta) &&
                    moesq_aligned16(sf),
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(out % 128 == 0 && K % 128 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  MOESQ_REQUIRE(kind == MOESQ_LINEAR_DOWN || out % 256 == 0, MOESQ_ERR_UNSUPPORTED_SHAPE);
  if (E * out == 0) return MOESQ_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t n1 = E * (out / 128) * ((K + 255) / 256) * 128;
  k_repack_meta<<<grid_for(n1, 128), 128, 0, s>>>(mask, E, out, K, kind != MOESQ_LINEAR_DOWN, meta,
                                                  d_status);
  MOESQ_CHECK_LAUNCH();
  const int64_t n2 = E * (out / 128) * (K / 128) * 32;
  int g2 = grid_for(n2, 128);
  if ((int64_t)g2 * 128 < E) g2 = (int)((E + 127) / 128);
  k_repack_sf<<<g2, 128, 0, s>>>(scale, g_w, E, out, K, kind, sf, alpha_w);
  MOESQ_CHECK_LAUNCH();
  return MOESQ_OK;
}
