// wpk_debug_gemm: one tensor-core tile, D[128][N] = A[128][K] . (B1 + B2)[N][K]^T,
// through the same path the program's tensor-core tiles use (bulk copies of
// swizzled operand images into a staging ring, tcgen05.mma with fp32
// accumulation in TMEM, tcgen05.ld epilogue).  Used by the tests to check the
// descriptor, swizzle and TMEM-lane conventions against a host matmul.
#include <cuda_runtime.h>

#include "mma.cuh"
#include "wpk_internal.h"

namespace wpk {
namespace {

constexpr int kDbgStages = 2;

__global__ void __launch_bounds__(128, 1)
    debug_gemm_kernel(const uint8_t* a, const uint8_t* b1, const uint8_t* b2, float* d, int n_chunks, int N,
                      int bf16, int* status) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t bars[2 * kDbgStages + 1];
  __shared__ uint32_t tmem_base;
  const int stage_bytes = kMmaABytes + 2 * N * 128;
  MmaRing R;
  R.base = smem;
  R.stage_bytes = stage_bytes;
  R.stages = kDbgStages;
  R.full = bars;
  R.empty = bars + kDbgStages;
  R.done = bars + 2 * kDbgStages;
  R.full_phase = R.empty_phase = R.done_phase = 0;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * kDbgStages + 1; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;
  uint32_t pend = 0;
  if (threadIdx.x == 0) {
    MmaJob J;
    J.a = a;
    J.b = b1;
    J.b2 = b2;
    J.b_chunk_bytes = N * 128;
    J.n_chunks = n_chunks;
    J.N = N;
    J.bf16 = bf16 != 0;
    ok = mma_run_issuer(R, J, tmem, 2000000000ull, &pend);
    if (!ok) atomicExch(status, 1);
  }
  ok = __syncthreads_and(ok);
  if (ok) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(R.done, 0))
      if (globaltimer() - t0 > 2000000000ull) {
        atomicExch(status, 2);
        ok = false;
        break;
      }
  }
  ok = __syncthreads_and(ok);
  tc_fence_after();
  if (ok) {
    const int row = warp * 32 + (threadIdx.x & 31);
    for (int c0 = 0; c0 < N; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) d[(size_t)row * N + c0 + i] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace
}  // namespace wpk

using namespace wpk;

extern "C" int wpk_debug_gemm(const void* a_img_dev, const void* b1_img_dev, const void* b2_img_dev, float* d_dev,
                              int n_chunks, int N, int bf16, void* stream) {
  if (!a_img_dev || !b1_img_dev || !d_dev || n_chunks <= 0 || N < 16 || N > 256 || N % 16) return WPK_ERR_INVALID_ARG;
  const size_t smem = (size_t)kDbgStages * (kMmaABytes + 2 * N * 128);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaFuncSetAttribute(debug_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return WPK_ERR_CUDA;
  int* status = nullptr;
  if (cudaMallocAsync(&status, 4, s) != cudaSuccess) return WPK_ERR_CUDA;
  cudaMemsetAsync(status, 0, 4, s);
  debug_gemm_kernel<<<1, 128, smem, s>>>(static_cast<const uint8_t*>(a_img_dev), static_cast<const uint8_t*>(b1_img_dev),
                                         static_cast<const uint8_t*>(b2_img_dev), d_dev, n_chunks, N, bf16, status);
  int h = 0;
  cudaMemcpyAsync(&h, status, 4, cudaMemcpyDeviceToHost, s);
  cudaStreamSynchronize(s);
  cudaFreeAsync(status, s);
  if (cudaGetLastError() != cudaSuccess) return WPK_ERR_CUDA;
  return h ? WPK_ERR_TIMEOUT : WPK_OK;
}
