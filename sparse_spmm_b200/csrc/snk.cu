// snk.cu -- the extern "C" boundary of libsnk.so (declared in include/snk.h).
// Host-side argument checks, device bookkeeping and dispatch only; every step of the
// layer runs in the kernels of format.cu and spmm.cu.
#include <new>

#include "internal.cuh"

namespace {

bool valid_dtype(int dt) { return dt == SNK_F32 || dt == SNK_BF16; }
int elem_bytes(snk_dtype dt) { return dt == SNK_F32 ? 4 : 2; }

// Runs `fn` with L's device current, restoring the caller's device afterwards.
template <typename Fn>
snk_status on_device(int device, Fn fn) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  if (cur == device) return fn();
  if (cudaSetDevice(device) != cudaSuccess) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  const snk_status st = fn();
  (void)cudaSetDevice(cur);
  return st;
}

}  // namespace

extern "C" {

const char* snk_status_string(snk_status s) {
  switch (s) {
    case SNK_OK: return "SNK_OK";
    case SNK_ERR_INVALID_ARG: return "SNK_ERR_INVALID_ARG";
    case SNK_ERR_OUT_OF_RANGE: return "SNK_ERR_OUT_OF_RANGE";
    case SNK_ERR_DUPLICATE: return "SNK_ERR_DUPLICATE";
    case SNK_ERR_WORKSPACE_TOO_SMALL: return "SNK_ERR_WORKSPACE_TOO_SMALL";
    case SNK_ERR_UNSUPPORTED: return "SNK_ERR_UNSUPPORTED";
    case SNK_ERR_INVALID_VALUE: return "SNK_ERR_INVALID_VALUE";
    case SNK_ERR_NO_ROOM: return "SNK_ERR_NO_ROOM";
    case SNK_ERR_TIMEOUT: return "SNK_ERR_TIMEOUT";
    case SNK_ERR_CUDA: return "SNK_ERR_CUDA";
  }
  return "SNK_ERR_UNKNOWN";
}

int32_t snk_default_num_parts(int64_t nnz, int32_t sm_count) {
  if (sm_count < 1) sm_count = 1;
  const int64_t by_size = (nnz + 255) / 256;
  int64_t p = std::min<int64_t>(3 * (int64_t)sm_count, by_size);
  return (int32_t)std::max<int64_t>(p, 1);
}

static bool sizes_ok(int64_t M, int64_t K, int64_t nnz) {
  if (M < 1 || K < 1 || nnz < 0) return false;
  if (M >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || nnz >= ((int64_t)1 << 31)) return false;
  if (M > (((int64_t)1 << 62) / K)) return false;
  return nnz <= M * K;
}

static int32_t effective_parts(int64_t nnz, int32_t P) {
  const int64_t cap = std::max<int64_t>(nnz, 1);
  return (int32_t)std::min<int64_t>(P, cap);
}

static snk_status resolve_parts(int64_t nnz, int32_t req, int32_t* P_out, int* sm_out) {
  int dev = 0, sms = 1;
  if (req == 0) {
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return SNK_ERR_CUDA;
    }
    req = snk_default_num_parts(nnz, sms);
  }
  if (req < 1) return SNK_ERR_INVALID_ARG;
  *P_out = effective_parts(nnz, req);
  if (sm_out) *sm_out = sms;
  return SNK_OK;
}

size_t snk_workspace_bytes(int64_t M, int64_t K, int64_t nnz, int32_t num_parts) {
  if (!sizes_ok(M, K, nnz) || num_parts < 0) return 0;
  int32_t P = 0;
  if (resolve_parts(nnz, num_parts, &P, nullptr) != SNK_OK) return 0;
  return snk::workspace_bytes(M, K, nnz, P);
}

snk_status snk_build(int64_t M, int64_t K, int64_t nnz, int32_t* row, int32_t* col, void* values, snk_dtype vdt,
                     int32_t num_parts, void* workspace, size_t ws_bytes, snk_stream stream, snk_layout** out) {
  if (out == nullptr) return SNK_ERR_INVALID_ARG;
  *out = nullptr;
  if (!sizes_ok(M, K, nnz)) {
    if (M >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || nnz >= ((int64_t)1 << 31)) return SNK_ERR_UNSUPPORTED;
    return SNK_ERR_INVALID_ARG;
  }
  if (!valid_dtype(vdt) || num_parts < 0 || workspace == nullptr) return SNK_ERR_INVALID_ARG;
  if (nnz > 0 && (row == nullptr || col == nullptr || values == nullptr)) return SNK_ERR_INVALID_ARG;
  int32_t P = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  int sms = 1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SNK_ERR_CUDA;
  }
  SNK_TRY(resolve_parts(nnz, num_parts, &P, nullptr));
  snk_layout* L = new (std::nothrow) snk_layout();
  if (L == nullptr) return SNK_ERR_CUDA;
  L->M = M;
  L->K = K;
  L->nnz = nnz;
  L->P = P;
  L->dtype = vdt;
  L->device = dev;
  L->sm_count = sms;
  L->row = row;
  L->col = col;
  L->index_bits = 32;
  snk_status st = snk::layout_carve(L, workspace, ws_bytes);
  if (st == SNK_OK) st = snk::build_format(L, values, elem_bytes(vdt), (cudaStream_t)stream);
  if (st != SNK_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SNK_OK;
}

static snk_status check_dense(const void* p, int64_t ld, int64_t N, int64_t rows) {
  if (ld < N) return SNK_ERR_INVALID_ARG;
  if (rows > 0 && N > 0 && p == nullptr) return SNK_ERR_INVALID_ARG;
  return SNK_OK;
}

snk_status snk_forward(const snk_layout* L, const void* values, const void* X, int64_t N, int64_t ldx, void* Y,
                       int64_t ldy, snk_dtype dt, snk_stream stream) {
  if (L == nullptr || dt != L->dtype || N < 0) return SNK_ERR_INVALID_ARG;
  if (N == 0) return SNK_OK;
  if (L->nnz > 0 && values == nullptr) return SNK_ERR_INVALID_ARG;
  SNK_TRY(check_dense(X, ldx, N, L->K));
  SNK_TRY(check_dense(Y, ldy, N, L->M));
  return on_device(L->device, [&] { return snk::launch_spmm(L, false, values, X, N, ldx, Y, ldy, (cudaStream_t)stream); });
}

snk_status snk_backward_input(const snk_layout* L, const void* values, const void* dY, int64_t N, int64_t lddy,
                              void* dX, int64_t lddx, snk_dtype dt, snk_stream stream) {
  if (L == nullptr || dt != L->dtype || N < 0) return SNK_ERR_INVALID_ARG;
  if (N == 0) return SNK_OK;
  if (L->nnz > 0 && values == nullptr) return SNK_ERR_INVALID_ARG;
  SNK_TRY(check_dense(dY, lddy, N, L->M));
  SNK_TRY(check_dense(dX, lddx, N, L->K));
  return on_device(L->device,
                   [&] { return snk::launch_spmm(L, true, values, dY, N, lddy, dX, lddx, (cudaStream_t)stream); });
}

snk_status snk_backward_weight(const snk_layout* L, const void* dY, int64_t lddy, const void* X, int64_t ldx,
                               int64_t N, void* dW, snk_dtype dt, snk_stream stream) {
  if (L == nullptr || dt != L->dtype || N < 0) return SNK_ERR_INVALID_ARG;
  if (N >= ((int64_t)1 << 31)) return SNK_ERR_UNSUPPORTED;
  if (L->nnz == 0) return SNK_OK;
  if (dW == nullptr) return SNK_ERR_INVALID_ARG;
  SNK_TRY(check_dense(dY, lddy, N, L->M));
  SNK_TRY(check_dense(X, ldx, N, L->K));
  return on_device(L->device,
                   [&] { return snk::launch_sddmm(L, dY, lddy, X, ldx, N, dW, (cudaStream_t)stream); });
}

snk_status snk_restructure(snk_layout* L, void* values, int64_t drop_count, uint64_t seed, float regrow_value,
                           int32_t* old_to_new, snk_stream stream) {
  if (L == nullptr || drop_count < 0) return SNK_ERR_INVALID_ARG;
  if (L->nnz > 0 && values == nullptr) return SNK_ERR_INVALID_ARG;
  return on_device(L->device, [&] {
    return snk::restructure(L, values, drop_count, seed, regrow_value, old_to_new, (cudaStream_t)stream);
  });
}

snk_status snk_remap_entries(const int32_t* old_to_new, int64_t nnz, const void* src, void* dst, int32_t elem_bytes,
                             snk_stream stream) {
  if (nnz < 0 || (elem_bytes != 2 && elem_bytes != 4)) return SNK_ERR_INVALID_ARG;
  if (nnz > 0 && (old_to_new == nullptr || src == nullptr || dst == nullptr || src == dst)) return SNK_ERR_INVALID_ARG;
  return snk::remap_entries(old_to_new, nnz, src, dst, elem_bytes, (cudaStream_t)stream);
}

snk_status snk_set_index_bits(snk_layout* L, int32_t bits) {
  if (L == nullptr || (bits != 16 && bits != 32)) return SNK_ERR_INVALID_ARG;
  if (bits == 16 && (L->col16 == nullptr || L->csc_row16 == nullptr)) return SNK_ERR_UNSUPPORTED;
  L->index_bits = bits;
  return SNK_OK;
}

snk_status snk_sync_status(snk_layout* L, snk_stream stream) {
  if (L == nullptr) return SNK_ERR_INVALID_ARG;
  return on_device(L->device, [&]() -> snk_status {
    const cudaStream_t s = (cudaStream_t)stream;
    uint32_t e = 0;
    SNK_CUDA_TRY(cudaMemcpyAsync(&e, L->err, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
    SNK_CUDA_TRY(cudaStreamSynchronize(s));
    if ((e & snk::ERRBIT_TIMEOUT) == 0) return SNK_OK;
    SNK_CUDA_TRY(cudaMemsetAsync(L->err, 0, sizeof(uint32_t), s));
    SNK_CUDA_TRY(cudaStreamSynchronize(s));
    return SNK_ERR_TIMEOUT;
  });
}

snk_status snk_layout_info(const snk_layout* L, snk_layout_view* v) {
  if (L == nullptr || v == nullptr) return SNK_ERR_INVALID_ARG;
  v->M = L->M;
  v->K = L->K;
  v->nnz = L->nnz;
  v->num_parts = L->P;
  v->dtype = (int32_t)L->dtype;
  v->device = L->device;
  v->row = L->row;
  v->col = L->col;
  v->row_ptr = L->row_ptr;
  v->col_ptr = L->col_ptr;
  v->csc_row = L->csc_row;
  v->perm = L->perm;
  v->part_nnz = L->part_nnz;
  v->part_row = L->part_row;
  v->part_nnz_t = L->part_nnz_t;
  v->part_col = L->part_col;
  return SNK_OK;
}

void snk_destroy(snk_layout* L) { delete L; }

}  // extern "C"
