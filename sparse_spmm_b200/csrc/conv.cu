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

// Each thread writes 4 consecutive patch columns (one 4-element vector store when the row
// is aligned); the image coordinates of the first come from two 32-bit divisions and the
// rest by stepping w, h, n.  The reads are element by element (shifted by kw - 1).
template <typename E>
__global__ void k_im2col3x3(const E* __restrict__ x, uint32_t Nb, uint32_t H, uint32_t W, E* __restrict__ out,
                            int64_t ld, bool vec) {
  const uint32_t r = blockIdx.y;  // ci*9 + k
  const uint32_t ci = r / 9, k = r % 9;
  const int kh = (int)(k / 3), kw = (int)(k % 3);
  const uint32_t HW = H * W, P = Nb * HW;
  const E* __restrict__ xc = x + (int64_t)ci * P;
  E* __restrict__ o = out + (int64_t)r * ld;
  for (uint32_t j0 = 4u * (blockIdx.x * blockDim.x + threadIdx.x); j0 < P; j0 += 4u * gridDim.x * blockDim.x) {
    uint32_t n = j0 / HW;
    const uint32_t rem = j0 - n * HW;
    uint32_t h = rem / W, w = rem - h * W;
    E v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int hs = (int)h + kh - 1, ws = (int)w + kw - 1;
      const bool in = j0 + q < P && hs >= 0 && hs < (int)H && ws >= 0 && ws < (int)W;
      v[q] = in ? xc[((int64_t)n * H + hs) * W + ws] : E(0);
      if (++w == W) {
        w = 0;
        if (++h == H) {
          h = 0;
          ++n;
        }
      }
    }
    if (vec && j0 + 4 <= P) {
      if constexpr (sizeof(E) == 4)
        *reinterpret_cast<uint4*>(o + j0) = make_uint4(v[0], v[1], v[2], v[3]);
      else
        *reinterpret_cast<uint2*>(o + j0) = make_uint2((uint32_t)v[0] | ((uint32_t)v[1] << 16),
                                                       (uint32_t)v[2] | ((uint32_t)v[3] << 16));
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (j0 + q < P) o[j0 + q] = v[q];
    }
  }
}

}  // namespace

extern "C" SNK_API snk_status snk_im2col3x3(const void* x, int64_t C, int64_t Nb, int64_t H, int64_t W, void* out,
                                            int64_t ld, snk_dtype dt, snk_stream stream) {
  if (C <= 0 || Nb <= 0 || H <= 0 || W <= 0 || x == nullptr || out == nullptr) return SNK_ERR_INVALID_ARG;
  if (dt != SNK_F32 && dt != SNK_BF16) return SNK_ERR_INVALID_ARG;
  const int64_t P = Nb * H * W;
  if (ld < P || 9 * C > 65535 || P >= ((int64_t)1 << 31) - 4) return SNK_ERR_INVALID_ARG;
  const int threads = 256;
  const dim3 grid((unsigned)std::min<int64_t>((P + 4 * threads - 1) / (4 * threads), 1024), (unsigned)(9 * C));
  const cudaStream_t s = (cudaStream_t)stream;
  const int elem = dt == SNK_F32 ? 4 : 2;
  const bool vec = ((uintptr_t)out % (4 * elem)) == 0 && (ld % 4) == 0;  // 4-element stores stay aligned
  if (dt == SNK_F32)
    k_im2col3x3<uint32_t><<<grid, threads, 0, s>>>((const uint32_t*)x, (uint32_t)Nb, (uint32_t)H, (uint32_t)W,
                                                   (uint32_t*)out, ld, vec);
  else
    k_im2col3x3<uint16_t><<<grid, threads, 0, s>>>((const uint16_t*)x, (uint32_t)Nb, (uint32_t)H, (uint32_t)W,
                                                   (uint16_t*)out, ld, vec);
  return cudaGetLastError() == cudaSuccess ? SNK_OK : SNK_ERR_CUDA;
}
