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

extern "C" moesq_status moesq_moe_forward_host_workspace_size(const moesq_moe_layer* L,
                                                              int64_t T, size_t* bytes) {
  if (!bytes || !L) return MOESQ_ERR_INVALID_ARG;
  size_t fw = 0;
  moesq_status st = moesq_moe_forward_workspace_size(L, T, &fw);
  if (st != MOESQ_OK) return st;
  const size_t io = align256((size_t)T * L->H * 2) * 2 + align256((size_t)T * L->k * 4) * 2;
  *bytes = align256(fw) + io;
  return MOESQ_OK;
}

extern "C" moesq_status moesq_moe_forward_host(const moesq_moe_layer* L, const uint16_t* h_x,
                                               const int32_t* h_topk_ids, const float* h_topk_w,
                                               int64_t T, uint16_t* h_out, void* ws,
                                               size_t ws_bytes, int32_t* d_status,
                                               moesq_stream_t stream) {
  size_t need = 0, fw = 0;
  moesq_status st = moesq_moe_forward_host_workspace_size(L, T, &need);
  if (st != MOESQ_OK) return st;
  moesq_moe_forward_workspace_size(L, T, &fw);
  if (T == 0) return MOESQ_OK;
  MOESQ_REQUIRE(h_x && h_topk_ids && h_topk_w && h_out, MOESQ_ERR_INVALID_ARG);
  MOESQ_REQUIRE(ws && ws_bytes >= need && moesq_aligned16(ws), MOESQ_ERR_WORKSPACE);
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* w = (uint8_t*)ws;
  size_t o = align256(fw);
  uint16_t* dx = (uint16_t*)(w + o);
  o += align256((size_t)T * L->H * 2);
  uint16_t* dout = (uint16_t*)(w + o);
  o += align256((size_t)T * L->H * 2);
  int32_t* dids = (int32_t*)(w + o);
  o += align256((size_t)T * L->k * 4);
  float* dw = (float*)(w + o);
  if (cudaMemcpyAsync(dx, h_x, (size_t)T * L->H * 2, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dids, h_topk_ids, (size_t)T * L->k * 4, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(dw, h_topk_w, (size_t)T * L->k * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  st = moesq_moe_forward(L, dx, dids, dw, T, dout, ws, fw, d_status, stream);
  if (st != MOESQ_OK) return st;
  if (cudaMemcpyAsync(h_out, dout, (size_t)T * L->H * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOESQ_ERR_CUDA;
  return MOESQ_OK;
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
