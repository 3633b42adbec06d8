// The rate of the sparse block-scaled FP4 tensor-core MMA on this device: the
// denominator of the grouped GEMMs' tensor roofline (the grouped GEMM is the kernel
// line of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card; its peak is taken as the
// larger of this measurement and 8 x the measured bf16 GEMM rate, the nominal sparse
// FP4 to dense bf16 ratio).
//
// Every SM pair issues back-to-back tcgen05.mma.sp.cta_group::2.kind::mxf4nvf4 with
// M = 256 and dense K = 128 on operands that sit in shared memory and TMEM from the
// start: no copies from global memory, so the time is the tensor core's alone
// (operand reads from shared memory included).  The operands are the grouped GEMM's
// stage layout: a 512-deep weight tile (SW128), the CTA's 128 token rows of two
// 256-deep chunks, sparse metadata selecting pairs 0 and 1 of every chunk of eight
// (a valid 4:8 pattern), unit E4M3 scales; the values are zero.
#include "common.cuh"

namespace moesq {
namespace peak {

constexpr int THREADS = 128;
constexpr int A_BYTES = 128 * 128;         // 128 weight rows x 512 dense K, compressed
constexpr int B_CHUNK = 128 * 128;         // 128 token rows x 256 dense K
constexpr int B_BYTES = 2 * B_CHUNK;
constexpr int E_BYTES = 2 * 128 * 16;      // metadata of 512 dense K
constexpr int SF_BYTES = 4 * 512;          // scale blocks of four MMAs
constexpr int OFF_E = A_BYTES + B_BYTES, OFF_SFA = OFF_E + E_BYTES, OFF_SFB = OFF_SFA + SF_BYTES;
constexpr int OPERAND_BYTES = OFF_SFB + 2 * SF_BYTES;
// more than half of an SM's shared memory, so that one CTA holds each SM (and its TMEM)
constexpr int SMEM_BYTES = 120 * 1024;
constexpr uint32_t TM_E = 384, TM_SFA = 392, TM_SFB = 408;
static_assert(OPERAND_BYTES + 1024 <= SMEM_BYTES, "operands");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_sparse_mma_peak(int iters, uint32_t n, int32_t* d_status) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  uint8_t* smem = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5;
  const bool lead = cluster_ctarank() == 0;
  for (int i = threadIdx.x; i < OPERAND_BYTES / 16; i += THREADS) {
    const int off = 16 * i;
    const uint32_t w = off < OFF_E ? 0u : off < OFF_SFA ? 0x44444444u : 0x38383838u;
    *reinterpret_cast<uint4*>(smem + off) = make_uint4(w, w, w, w);
  }
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base, 512);
    tmem_relinquish_pair();
  }
  fence_proxy_async_smem();  // the operands, written by threads, are read by the tensor core
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (lead && warp == 1 && elect_one()) {
    const uint32_t s0 = smem_u32(smem);
    const uint64_t dA = smem_desc(s0, 16, 1024, SWZ_128B);
    const uint64_t dB = smem_desc(s0 + A_BYTES, 16, 1024, SWZ_128B);
    const uint64_t dE = smem_desc(s0 + OFF_E, 128 * 16, 128, SWZ_NONE);
    const uint64_t dSFA = smem_desc(s0 + OFF_SFA, 16, 128, SWZ_NONE);
    const uint64_t dSFB = smem_desc(s0 + OFF_SFB, 16, 128, SWZ_NONE);
    tc_cp_pair_128x256b(tmem + TM_E, dE);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tc_cp_pair_32x128b_warpx4(tmem + TM_SFA + 4 * j, dSFA + (uint64_t)(j * (512 >> 4)));
      tc_cp_pair_32x128b_warpx4(tmem + TM_SFB + 8 * j, dSFB + (uint64_t)(j * (512 >> 4)));
      tc_cp_pair_32x128b_warpx4(tmem + TM_SFB + 8 * j + 4, dSFB + (uint64_t)((SF_BYTES + j * 512) >> 4));
    }
    const uint32_t idesc = (1u << 2) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((256u >> 4) << 24);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tc_mma_pair_sp_nvf4(tmem, dA + (uint64_t)(j * 2), dB + (uint64_t)((j >> 1) * (B_CHUNK >> 4) + (j & 1) * 4),
                            tmem + TM_E + 2 * j, idesc, tmem + TM_SFA + 4 * j, tmem + TM_SFB + 8 * j,
                            (it > 0 || j > 0) ? 1u : 0u);
    }
    tc_commit_pair_mc(&done, 0x3);
  }
  __syncwarp();
  mbar_wait_spin(&done, 0, &abort_flag, d_status);  // bounded; flags a timeout
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace peak
}  // namespace moesq

using namespace moesq;

extern "C" moesq_status moesq_measure_sparse_mma_peak(int32_t iters, int32_t n, double* tflops, int32_t* d_status,
                                                      moesq_stream_t stream) {
  MOESQ_REQUIRE(tflops && iters >= 1 && n >= 16 && n <= 256 && n % 16 == 0, MOESQ_ERR_INVALID_ARG);
  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  if (major != 10) return MOESQ_ERR_DEVICE;
  if (cudaFuncSetAttribute(peak::k_sparse_mma_peak, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           peak::SMEM_BYTES) != cudaSuccess)
    return MOESQ_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid((unsigned)(sms & ~1));
  cudaEvent_t a = nullptr, b = nullptr;
  if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return MOESQ_ERR_CUDA;
  moesq_status rc = MOESQ_OK;
  float ms = 0.0f;
  // one warm-up launch, then the timed one
  for (int rep = 0; rep < 2 && rc == MOESQ_OK; ++rep) {
    if (rep == 1 && cudaEventRecord(a, st) != cudaSuccess) rc = MOESQ_ERR_CUDA;
    if (rc == MOESQ_OK && moesq_launch(peak::k_sparse_mma_peak, grid, dim3(peak::THREADS), peak::SMEM_BYTES, st,
                                       iters, (uint32_t)n, d_status) != cudaSuccess)
      rc = MOESQ_ERR_CUDA;
  }
  if (rc == MOESQ_OK && (cudaEventRecord(b, st) != cudaSuccess || cudaEventSynchronize(b) != cudaSuccess ||
                         cudaEventElapsedTime(&ms, a, b) != cudaSuccess))
    rc = MOESQ_ERR_CUDA;
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (rc != MOESQ_OK) {
    (void)cudaGetLastError();
    return rc;
  }
  // dense-equivalent FLOPs: 2 M N K per MMA, M = 256 per pair, dense K = 128
  const double flops = 2.0 * 256.0 * n * 128.0 * 4.0 * iters * (double)(grid.x / 2);
  *tflops = ms > 0.0f ? flops / (ms * 1e-3) / 1e12 : 0.0;
  return MOESQ_OK;
}
