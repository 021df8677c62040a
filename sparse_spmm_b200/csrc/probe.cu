// FP32 FMA-rate probe: the ALU roofline of the products at large N (no part of the method).

#include <cuda_runtime.h>

#include "internal.cuh"
#include "snk.h"

namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeChains = 8;  // independent packed chains per thread

// Each thread runs kProbeChains independent chains of packed fp32 FMAs (two FMAs per
// instruction), iters steps each; the sum is written so that nothing is dead code.
__global__ void __launch_bounds__(kProbeThreads) k_fma_rate(float* sink, int iters, float m) {
  float2 a[kProbeChains];
#pragma unroll
  for (int j = 0; j < kProbeChains; ++j) a[j] = make_float2(threadIdx.x * 1e-3f + j, j * 1e-3f);
  const float2 mm = make_float2(m, m), cc = make_float2(1e-7f, -1e-7f);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int j = 0; j < kProbeChains; ++j) a[j] = __ffma2_rn(a[j], mm, cc);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < kProbeChains; ++j) s += a[j].x + a[j].y;
  if (s == 1234.5f) sink[blockIdx.x] = s;  // practically never taken; keeps the chains live
}

}  // namespace

extern "C" SNK_API snk_status snk_probe_fp32_fma(int32_t blocks, int32_t iters, float* sink, snk_stream stream) {
  if (blocks <= 0 || iters <= 0 || sink == nullptr) return SNK_ERR_INVALID_ARG;
  k_fma_rate<<<blocks, kProbeThreads, 0, (cudaStream_t)stream>>>(sink, iters, 0.999999f);
  return cudaGetLastError() == cudaSuccess ? SNK_OK : SNK_ERR_CUDA;
}

extern "C" SNK_API int64_t snk_probe_fp32_fma_flops(int32_t blocks, int32_t iters) {
  return (int64_t)blocks * kProbeThreads * iters * kProbeChains * 2 * 2;
}
