// conv.cu -- the patch matrix ("im2col") of a 3x3 convolution, so that a sparse 3x3 layer
// runs as the forward SpMM with K = 9 C ("SparseRT: Accelerating Unstructured Sparsity on
// GPUs for Deep Learning Inference", Abstract: sparse 1x1 and 3x3 convolutions).
//
// out[(ci*9 + kh*3 + kw)][(n*H + h)*W + w] = x[ci][n][h+kh-1][w+kw-1], zero outside the
// image (stride 1, zero padding 1).  The row index is the flattening of a [Co][C][3][3]
// weight, so W's column index is ci*9 + kh*3 + kw.  Pure data movement: each element is
// copied bit for bit.  One CTA row per patch-matrix row, threads along the columns, so the
// writes are coalesced and the reads are too, up to the one-element shift.
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.cuh"
#include "snk.h"

namespace {

template <typename E>
__global__ void k_im2col3x3(const E* __restrict__ x, int64_t C, int64_t Nb, int64_t H, int64_t W,
                            E* __restrict__ out, int64_t ld) {
  const int64_t r = blockIdx.y;  // ci*9 + k
  const int64_t ci = r / 9, k = r % 9, kh = k / 3, kw = k % 3;
  const int64_t P = Nb * H * W, HW = H * W;
  const E* __restrict__ xc = x + ci * P;
  E* __restrict__ o = out + r * ld;
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < P; j += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = j / HW, rem = j - n * HW, h = rem / W, w = rem - h * W;
    const int64_t hs = h + kh - 1, ws = w + kw - 1;
    o[j] = (hs >= 0 && hs < H && ws >= 0 && ws < W) ? xc[(n * H + hs) * W + ws] : E(0);
  }
}

}  // namespace

extern "C" SNK_API snk_status snk_im2col3x3(const void* x, int64_t C, int64_t Nb, int64_t H, int64_t W, void* out,
                                            int64_t ld, snk_dtype dt, snk_stream stream) {
  if (C <= 0 || Nb <= 0 || H <= 0 || W <= 0 || x == nullptr || out == nullptr) return SNK_ERR_INVALID_ARG;
  if (dt != SNK_F32 && dt != SNK_BF16) return SNK_ERR_INVALID_ARG;
  const int64_t P = Nb * H * W;
  if (ld < P || 9 * C > 65535) return SNK_ERR_INVALID_ARG;
  const int threads = 256;
  const dim3 grid((unsigned)std::min<int64_t>((P + threads - 1) / threads, 1024), (unsigned)(9 * C));
  const cudaStream_t s = (cudaStream_t)stream;
  if (dt == SNK_F32)
    k_im2col3x3<uint32_t><<<grid, threads, 0, s>>>((const uint32_t*)x, C, Nb, H, W, (uint32_t*)out, ld);
  else
    k_im2col3x3<uint16_t><<<grid, threads, 0, s>>>((const uint16_t*)x, C, Nb, H, W, (uint16_t*)out, ld);
  return cudaGetLastError() == cudaSuccess ? SNK_OK : SNK_ERR_CUDA;
}
