// Status strings and the whole routed-expert MLP (moesq_moe_forward).
//
// moe_forward chains the library's own kernels on one stream, with no host
// synchronisation: permute -> quant_act (gather + per-expert global, padded
// operand layout) -> gate_up grouped GEMM with the fused SwiGLU + NVFP4
// requant epilogue -> down grouped GEMM (bf16 per slot) -> weighted combine.
// The expert MLP is gate_proj/up_proj/down_proj of the routed experts ("Compressed
// layers" row of the "Compression details" table, Qwen3.5-397B-A17B-P48NVFP4-
// MoESQ model card).
#include "common.cuh"

#include <mutex>

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct FwdLayout {
  size_t off_expert, off_pad, off_slot_token, off_token_slot, off_perm, off_a_codes, off_a_sf,
      off_h_codes, off_h_sf, off_y, total;
  int64_t S, P;
};

moesq_status fwd_layout(const moesq_moe_layer* L, int64_t T, FwdLayout* f) {
  if (!L || T < 0 || L->E < 1 || L->k < 1 || L->H <= 0 || L->I <= 0) return MOESQ_ERR_INVALID_ARG;
  if (L->H % 128 || L->I % 128) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  f->S = T * L->k;
  f->P = moesq_padded_rows(f->S, L->E);
  size_t perm = 0;
  moesq_status st = moesq_permute_workspace_size(T, L->k, L->E, &perm);
  if (st != MOESQ_OK) return st;
  size_t o = 0;
  f->off_expert = o;
  o = align256(o + (L->E + 1) * 4);
  f->off_pad = o;
  o = align256(o + (L->E + 1) * 4);
  f->off_slot_token = o;
  o = align256(o + f->S * 4);
  f->off_token_slot = o;
  o = align256(o + f->S * 4);
  f->off_perm = o;
  o = align256(o + perm);
  f->off_a_codes = o;
  o = align256(o + (size_t)f->P * (L->H / 2));
  f->off_a_sf = o;
  o = align256(o + (size_t)(f->P / 128) * (L->H / 128) * 512);
  f->off_h_codes = o;
  o = align256(o + (size_t)f->P * (L->I / 2));
  f->off_h_sf = o;
  o = align256(o + (size_t)(f->P / 128) * (L->I / 128) * 512);
  f->off_y = o;
  o = align256(o + (size_t)f->S * L->H * 2);
  f->total = o;
  return MOESQ_OK;
}

}  // namespace

extern "C" const char* moesq_status_string(int status) {
  switch (status) {
    case MOESQ_OK: return "ok";
    case MOESQ_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or enum, misaligned pointer)";
    case MOESQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOESQ_ERR_BAD_SPARSITY: return "paired-4:8 sparsity violated";
    case MOESQ_ERR_CUDA: return "CUDA runtime or driver call failed";
    case MOESQ_ERR_TIMEOUT: return "a bounded device wait gave up";
    case MOESQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MOESQ_ERR_DEVICE: return "current device is not sm_100";
    case MOESQ_ERR_CAPACITY: return "request exceeds the fixed scratch of an allocation-free entry point";
    default: return "unknown status";
  }
}

extern "C" int moesq_abi_version(void) { return 1; }

extern "C" moesq_status moesq_moe_forward_workspace_size(const moesq_moe_layer* L, int64_t T,
                                                         size_t* bytes) {
  if (!bytes) return MOESQ_ERR_INVALID_ARG;
  FwdLayout f;
  moesq_status st = fwd_layout(L, T, &f);
  if (st != MOESQ_OK) return st;
  *bytes = f.total;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_moe_forward(const moesq_moe_layer* L, const uint16_t* x,
                                          const int32_t* topk_ids, const float* topk_w, int64_t T,
                                          uint16_t* out, void* ws, size_t ws_bytes,
                                          int32_t* d_status, moesq_stream_t stream) {
  FwdLayout f;
  moesq_status st = fwd_layout(L, T, &f);
  if (st != MOESQ_OK) return st;
  if (T == 0) return MOESQ_OK;
  MOESQ_REQUIRE(x && topk_ids && topk_w && out, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(L->g_in_gate_up && L->g_in_down, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(L->gate_up.E == L->E && L->down.E == L->E, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(L->gate_up.out == 2 * L->I && L->gate_up.K == L->H && L->down.out == L->H &&
                    L->down.K == L->I,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(L->gate_up.kind != MOESQ_LINEAR_DOWN && L->down.kind == MOESQ_LINEAR_DOWN,
                MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(ws && ws_bytes >= f.total && moesq_aligned16(ws), MOESQ_ERR_WORKSPACE);
  uint8_t* w = (uint8_t*)ws;
  int32_t* eo = (int32_t*)(w + f.off_expert);
  int32_t* po = (int32_t*)(w + f.off_pad);
  int32_t* slot_token = (int32_t*)(w + f.off_slot_token);
  int32_t* token_slot = (int32_t*)(w + f.off_token_slot);
  uint8_t* a_codes = w + f.off_a_codes;
  uint8_t* a_sf = w + f.off_a_sf;
  uint8_t* h_codes = w + f.off_h_codes;
  uint8_t* h_sf = w + f.off_h_sf;
  uint16_t* y = (uint16_t*)(w + f.off_y);
  size_t perm_bytes = f.off_a_codes - f.off_perm;

  st = moesq_permute(topk_ids, T, L->k, L->E, eo, po, slot_token, token_slot, w + f.off_perm,
                     perm_bytes, d_status, stream);
  if (st != MOESQ_OK) return st;
  st = moesq_quant_act_routed(x, T, L->H, topk_ids, token_slot, L->k, eo, po, L->E, L->g_in_gate_up,
                              a_codes, a_sf, stream);
  if (st != MOESQ_OK) return st;
  st = moesq_grouped_gemm(&L->gate_up, a_codes, a_sf, L->g_in_gate_up, eo, po, f.S, f.P,
                          MOESQ_EPI_SWIGLU_NVFP4, L->g_in_down, h_codes, h_sf, nullptr, 0, d_status,
                          stream);
  if (st != MOESQ_OK) return st;
  st = moesq_grouped_gemm(&L->down, h_codes, h_sf, L->g_in_down, eo, po, f.S, f.P, MOESQ_EPI_BF16,
                          nullptr, y, nullptr, nullptr, 0, d_status, stream);
  if (st != MOESQ_OK) return st;
  return moesq_unpermute(y, token_slot, topk_w, T, L->k, L->H, out, stream);
}

// ------------------------------------------------------------- host forward --
// The batch is cut into token chunks whose host->device copies, forward and
// device->host copies overlap: uploads run on one internal stream, the forward on
// the caller's stream, downloads on a second internal stream, ordered by events.
// Each token's result depends only on its own row and routing, so the chunked
// forward equals the whole-batch one bit for bit.
namespace {

constexpr int64_t HOST_MIN_CHUNK = 2048;   // tokens: smaller chunks cost GEMM efficiency
constexpr int64_t HOST_MAX_CHUNKS = 8;     // each chunk has its own device buffers

int64_t host_chunk_tokens(int64_t T) {
  int64_t c = (T + HOST_MAX_CHUNKS - 1) / HOST_MAX_CHUNKS;
  if (c < HOST_MIN_CHUNK) c = HOST_MIN_CHUNK;
  return c < T ? c : T;
}

struct HostBufs {
  size_t x_bytes, idw_bytes, set_bytes, fw;
};

moesq_status host_layout(const moesq_moe_layer* L, int64_t T, HostBufs* h) {
  const int64_t tc = host_chunk_tokens(T);
  size_t fw = 0;
  moesq_status st = moesq_moe_forward_workspace_size(L, tc, &fw);
  if (st != MOESQ_OK) return st;
  h->fw = align256(fw);
  h->x_bytes = align256((size_t)tc * L->H * 2);
  h->idw_bytes = align256((size_t)tc * L->k * 4);
  h->set_bytes = 2 * h->x_bytes + 2 * h->idw_bytes;  // x, out, ids, weights
  return MOESQ_OK;
}

// the two copy streams of each device, created on first use and kept for the process
std::mutex g_copy_mu;
cudaStream_t g_copy_streams[64][2] = {};

cudaError_t copy_streams(cudaStream_t* up, cudaStream_t* down) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_copy_mu);
  for (int i = 0; i < 2; ++i)
    if (!g_copy_streams[dev][i]) {
      e = cudaStreamCreateWithFlags(&g_copy_streams[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) return e;
    }
  *up = g_copy_streams[dev][0];
  *down = g_copy_streams[dev][1];
  return cudaSuccess;
}

}  // namespace

extern "C" moesq_status moesq_moe_forward_host_workspace_size(const moesq_moe_layer* L,
                                                              int64_t T, size_t* bytes) {
  if (!bytes || !L || T < 0) return MOESQ_ERR_INVALID_ARG;
  HostBufs h;
  moesq_status st = host_layout(L, T > 0 ? T : 1, &h);
  if (st != MOESQ_OK) return st;
  const int64_t tc = host_chunk_tokens(T > 0 ? T : 1);
  const int64_t nsets = T > 0 ? (T + tc - 1) / tc : 1;
  *bytes = h.fw + (size_t)nsets * h.set_bytes;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_moe_forward_host(const moesq_moe_layer* L, const uint16_t* h_x,
                                               const int32_t* h_topk_ids, const float* h_topk_w,
                                               int64_t T, uint16_t* h_out, void* ws,
                                               size_t ws_bytes, int32_t* d_status,
                                               moesq_stream_t stream) {
  size_t need = 0;
  moesq_status st = moesq_moe_forward_host_workspace_size(L, T, &need);
  if (st != MOESQ_OK) return st;
  if (T == 0) return MOESQ_OK;
  MOESQ_REQUIRE(h_x && h_topk_ids && h_topk_w && h_out, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(ws && ws_bytes >= need && moesq_aligned16(ws), MOESQ_ERR_WORKSPACE);
  HostBufs hb;
  host_layout(L, T, &hb);
  const int64_t tc = host_chunk_tokens(T);
  const int64_t nchunks = (T + tc - 1) / tc;  // <= HOST_MAX_CHUNKS, one buffer set each
  cudaStream_t s = (cudaStream_t)stream, up = nullptr, down = nullptr;
  if (copy_streams(&up, &down) != cudaSuccess) return MOESQ_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  void* fws = w;
  // events: [chunk][0] uploaded, [chunk][1] computed; plus the entry point
  cudaEvent_t ev[HOST_MAX_CHUNKS][2] = {}, start = nullptr;
  moesq_status ret = MOESQ_OK;
  auto fail = [&](moesq_status code) {
    if (ret == MOESQ_OK) ret = code;
  };
  if (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess) return MOESQ_ERR_CUDA;
  for (int64_t c = 0; c < nchunks && ret == MOESQ_OK; ++c)
    for (int j = 0; j < 2; ++j)
      if (cudaEventCreateWithFlags(&ev[c][j], cudaEventDisableTiming) != cudaSuccess) fail(MOESQ_ERR_CUDA);
  // the copies start after the work already queued on the caller's stream
  if (ret == MOESQ_OK && (cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(up, start, 0) != cudaSuccess))
    fail(MOESQ_ERR_CUDA);
  for (int64_t c = 0; c < nchunks && ret == MOESQ_OK; ++c) {
    const int64_t t0 = c * tc, n = (T - t0) < tc ? (T - t0) : tc;
    uint8_t* set = w + hb.fw + (size_t)c * hb.set_bytes;
    uint16_t* dx = (uint16_t*)set;
    uint16_t* dout = (uint16_t*)(set + hb.x_bytes);
    int32_t* dids = (int32_t*)(set + 2 * hb.x_bytes);
    float* dw = (float*)(set + 2 * hb.x_bytes + hb.idw_bytes);
    if (cudaMemcpyAsync(dx, h_x + t0 * L->H, (size_t)n * L->H * 2, cudaMemcpyHostToDevice, up) != cudaSuccess ||
        cudaMemcpyAsync(dids, h_topk_ids + t0 * L->k, (size_t)n * L->k * 4, cudaMemcpyHostToDevice, up) !=
            cudaSuccess ||
        cudaMemcpyAsync(dw, h_topk_w + t0 * L->k, (size_t)n * L->k * 4, cudaMemcpyHostToDevice, up) !=
            cudaSuccess ||
        cudaEventRecord(ev[c][0], up) != cudaSuccess || cudaStreamWaitEvent(s, ev[c][0], 0) != cudaSuccess) {
      fail(MOESQ_ERR_CUDA);
      break;
    }
    st = moesq_moe_forward(L, dx, dids, dw, n, dout, fws, hb.fw, d_status, stream);
    if (st != MOESQ_OK) {
      fail(st);
      break;
    }
    if (cudaEventRecord(ev[c][1], s) != cudaSuccess || cudaStreamWaitEvent(down, ev[c][1], 0) != cudaSuccess ||
        cudaMemcpyAsync(h_out + t0 * L->H, dout, (size_t)n * L->H * 2, cudaMemcpyDeviceToHost, down) !=
            cudaSuccess) {
      fail(MOESQ_ERR_CUDA);
      break;
    }
  }
  // whatever was queued completes before the caller's buffers are handed back
  if (cudaStreamSynchronize(up) != cudaSuccess) fail(MOESQ_ERR_CUDA);
  if (cudaStreamSynchronize(s) != cudaSuccess) fail(MOESQ_ERR_CUDA);
  if (cudaStreamSynchronize(down) != cudaSuccess) fail(MOESQ_ERR_CUDA);
  for (int c = 0; c < HOST_MAX_CHUNKS; ++c)
    for (int j = 0; j < 2; ++j)
      if (ev[c][j]) cudaEventDestroy(ev[c][j]);
  if (start) cudaEventDestroy(start);
  return ret;
}

// ----------------------------------------------------------------- self-test --
// The bounded-wait failure path, exercised without a fault: thread 0 runs each of
// the library's three pipeline waits (suspending, spinning, polling) on an mbarrier
// phase that nothing completes.  Each gives up after limit_ns, ORs
// MOESQ_DFLAG_TIMEOUT into the status word and reports it; the kernel then
// returns normally and the context stays usable.
namespace {
__global__ void k_wait_timeout_selftest(int32_t* d_status, uint64_t limit_ns, int32_t* gave_up) {
  __shared__ uint64_t bar[3];
  __shared__ int abort_flag[3];
  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) {
      moesq::mbar_init(&bar[i], 1);
      abort_flag[i] = 0;
    }
    moesq::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 of a fresh barrier completes on one arrival, which never comes
    gave_up[0] = moesq::mbar_wait(&bar[0], 0, &abort_flag[0], d_status, limit_ns) ? 0 : 1;
    gave_up[1] = moesq::mbar_wait_spin(&bar[1], 0, &abort_flag[1], d_status, limit_ns) ? 0 : 1;
    gave_up[2] = moesq::mbar_wait_poll(&bar[2], 0, &abort_flag[2], d_status, limit_ns) ? 0 : 1;
  }
}
}  // namespace

extern "C" moesq_status moesq_selftest_wait_timeout(int32_t* d_status, int64_t limit_ns, int32_t* d_gave_up,
                                                    moesq_stream_t stream) {
  MOESQ_REQUIRE(d_status && d_gave_up && limit_ns > 0 && limit_ns <= 100000000, MOESQ_ERR_INVALID_ARG);
  k_wait_timeout_selftest<<<1, 32, 0, (cudaStream_t)stream>>>(d_status, (uint64_t)limit_ns, d_gave_up);
  return cudaGetLastError() == cudaSuccess ? MOESQ_OK : MOESQ_ERR_CUDA;
}
