// noalloc.cu -- snk_csr_forward_static: the forward product Y = W X for callers that
// cannot allocate device memory.
//
// Every other call of this library works on a layout whose device workspace the caller
// allocated (snk_workspace_bytes + a buffer of that size).  Some callers have no way to do
// that: code handed a CSR matrix by a host framework that owns all device memory and
// offers no allocator, plugins that may only use the buffers they are given, or code
// running where allocation is not permitted.  This entry point takes a plain CSR matrix
// (row pointers, column indices, values) plus X and Y, and allocates nothing: the few
// hundred kilobytes of scratch the forward kernel needs (per-CTA work descriptors, the
// fp32 carry slots of rows split between CTAs, their arrival counters) live in one
// file-scope __device__ array of fixed size, which every GPU that loads the library holds
// until the process exits.
#include <mutex>

#include "internal.cuh"

namespace {

// Capacity of the static scratch: at most kStaticMaxParts CTAs per launch.
constexpr int kStaticMaxParts = SNK_STATIC_MAX_PARTS;
constexpr size_t kDescBytes = sizeof(int4) * kStaticMaxParts;
constexpr size_t kCarryBytes = sizeof(float) * kStaticMaxParts * snk::kCarryCols;
constexpr size_t kCntBytes = sizeof(uint32_t) * kStaticMaxParts * snk::kMaxTiles;
constexpr size_t kScratchBytes = kDescBytes + 2 * kCarryBytes + kCntBytes;

// The scratch array itself.  In host code its name is only a stand-in: its device address
// is obtained with cudaGetSymbolAddress (once per device) and passed to the kernels.
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of g_static_scratch on `device` (which must be current).  The first call
// on a device resolves it; later calls return the cached address.
cudaError_t scratch_address(int device, unsigned char** out) {
  std::call_once(g_once[device], [device] {
    void* p = nullptr;
    g_scratch_err[device] = cudaGetSymbolAddress(&p, g_static_scratch);
    g_scratch_ptr[device] = p;
  });
  *out = static_cast<unsigned char*>(g_scratch_ptr[device]);
  return g_scratch_err[device];
}

__device__ __forceinline__ int64_t row_holding(const int32_t* __restrict__ ptr, int64_t dim, int64_t x) {
  int64_t lo = 0, hi = dim - 1;  // last r in [0, dim - 1] with ptr[r] <= x
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (ptr[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Clears the arrival counters (they must start at zero; a call may follow any earlier
// one) and writes the per-CTA work descriptors of P nnz-balanced parts: part p's range
// [floor(p nnz / P), floor((p+1) nnz / P)) with its ends moved to row boundaries where the
// row there is no longer than the smallest part (the same rule as the layout build).
__global__ void k_static_prepare(const int32_t* __restrict__ row_ptr, int64_t M, int64_t nnz, int P,
                                 int4* __restrict__ desc, uint32_t* __restrict__ cnt, int64_t ncnt) {
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = tid; i < ncnt; i += stride) cnt[i] = 0u;
  for (int64_t p = tid; p < P; p += stride) {
    const int64_t a = (p * nnz) / P, b = ((p + 1) * nnz) / P;
    const int64_t lmax = nnz / P;
    int64_t a2 = a, b2 = b;
    if (a < b) {
      const int64_t ra = row_holding(row_ptr, M, a);
      if (row_ptr[ra] < a && row_ptr[ra + 1] - row_ptr[ra] <= lmax) a2 = row_ptr[ra + 1];
      const int64_t t = row_holding(row_ptr, M, b - 1);
      if (row_ptr[t + 1] > b && row_ptr[t + 1] - row_ptr[t] <= lmax) b2 = row_ptr[t + 1];
      if (a2 > b2) a2 = b2;
    }
    const int64_t ra2 = a2 < nnz ? row_holding(row_ptr, M, a2) : M;
    const int64_t rb2 = b2 < nnz ? row_holding(row_ptr, M, b2) : M;
    desc[p] = make_int4((int)a2, (int)b2, (int)ra2, (int)rb2);
  }
}

}  // namespace

extern "C" snk_status snk_csr_forward_static(int64_t M, int64_t K, int64_t nnz, const int32_t* row_ptr,
                                             const int32_t* col, const void* values, snk_dtype dt, const void* X,
                                             int64_t N, int64_t ldx, void* Y, int64_t ldy, int32_t num_parts,
                                             snk_stream stream) {
  if (M < 1 || K < 1 || nnz < 0 || N < 0 || num_parts < 0) return SNK_ERR_INVALID_ARG;
  if (M >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || nnz >= ((int64_t)1 << 31)) return SNK_ERR_UNSUPPORTED;
  if (nnz > M * K) return SNK_ERR_INVALID_ARG;
  if (dt != SNK_F32 && dt != SNK_BF16) return SNK_ERR_INVALID_ARG;
  if (num_parts > kStaticMaxParts) return SNK_ERR_UNSUPPORTED;  // beyond the static scratch
  if (N == 0) return SNK_OK;
  if (ldx < N || ldy < N || X == nullptr || Y == nullptr || row_ptr == nullptr) return SNK_ERR_INVALID_ARG;
  if (nnz > 0 && (col == nullptr || values == nullptr)) return SNK_ERR_INVALID_ARG;

  int dev = 0, sms = 1;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SNK_ERR_UNSUPPORTED;
  unsigned char* base = nullptr;
  if (scratch_address(dev, &base) != cudaSuccess || base == nullptr) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  int64_t P = num_parts > 0 ? num_parts : snk_default_num_parts(nnz, sms);
  P = std::min<int64_t>(std::min<int64_t>(P, kStaticMaxParts), std::max<int64_t>(nnz, 1));

  snk_layout L{};
  L.M = M;
  L.K = K;
  L.nnz = nnz;
  L.P = (int32_t)P;
  L.dtype = dt;
  L.device = dev;
  L.sm_count = sms;
  L.row_ptr = const_cast<int32_t*>(row_ptr);
  L.col = const_cast<int32_t*>(col);
  L.desc_f = reinterpret_cast<int4*>(base);
  L.carry_tail_f = reinterpret_cast<float*>(base + kDescBytes);
  L.carry_head_f = reinterpret_cast<float*>(base + kDescBytes + kCarryBytes);
  L.cnt_f = reinterpret_cast<uint32_t*>(base + kDescBytes + 2 * kCarryBytes);
  cudaStream_t s = (cudaStream_t)stream;
  if (nnz > 0) {
    const int64_t ncnt = (int64_t)snk::kMaxTiles * P;
    k_static_prepare<<<(unsigned)((std::max<int64_t>(ncnt, P) + 255) / 256), 256, 0, s>>>(row_ptr, M, nnz, (int)P,
                                                                                          L.desc_f, L.cnt_f, ncnt);
    SNK_CUDA_TRY(cudaGetLastError());
  }
  return snk::launch_spmm(&L, false, values, X, N, ldx, Y, ldy, s);
}
