// internal.cuh -- shared definitions of the CUDA library (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "snk.h"

namespace snk {

// Device status word bits (OR-ed by kernels, read by the host after a sync).
enum : uint32_t {
  ERRBIT_OUT_OF_RANGE = 1u,
  ERRBIT_DUPLICATE = 2u,
  ERRBIT_INVALID_VALUE = 4u,
  ERRBIT_TIMEOUT = 8u,  // a bounded wait of a product kernel gave up
};

// Columns covered by one launch of the small-N SpMM kernels; the cross-CTA carry slots
// and the per-tile arrival counters are sized for this many columns.
constexpr int kCarryCols = 64;
constexpr int kMaxTiles = 64;

// Radix-sort tile: 256 threads x 8 keys.
constexpr int kSortThreads = 256;
constexpr int kSortItems = 8;
constexpr int kSortTile = kSortThreads * kSortItems;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Capacity of the sort buffers: the restructure merge needs nnz + drop_count <= 2 nnz,
// the regrowth rounds need (accepted < nnz) + (a batch >= nnz + 4096).
inline int64_t sort_capacity(int64_t nnz) { return 2 * nnz + 4096; }

// Index arrays fit 16 bits when both dimensions do.
inline bool index16_possible(int64_t M, int64_t K) { return M <= 65536 && K <= 65536; }

}  // namespace snk

// Host object behind snk_layout.  All pointers are device pointers into the caller's
// workspace except row/col, which are the caller's COO arrays.
struct snk_layout {
  int64_t M, K, nnz;
  int32_t P;
  snk_dtype dtype;
  int device;
  int sm_count;
  int32_t* row;
  int32_t* col;
  int32_t* row_ptr;
  int32_t* col_ptr;
  int32_t* csc_row;
  int32_t* perm;
  // 16-bit copies of col and csc_row (null unless M, K <= 65536), and the width the
  // products read (32 unless switched with snk_set_index_bits)
  uint16_t* col16;
  uint16_t* csc_row16;
  int index_bits;
  int32_t* part_nnz;
  int32_t* part_row;
  int32_t* part_nnz_t;
  int32_t* part_col;
  // per-CTA work descriptors of the products, one int4 per part: {a, b, ra, rb} = the
  // entry range the CTA walks and the rows holding a and b (see k_part_desc).
  int4* desc_f;
  int4* desc_t;
  // cross-CTA carries of the forward / transposed kernels: [P][kCarryCols] tail and head
  // slots, and [kMaxTiles][P] arrival counters (zero between launches).
  float* carry_tail_f;
  float* carry_head_f;
  uint32_t* cnt_f;
  float* carry_tail_b;
  float* carry_head_b;
  uint32_t* cnt_b;
  uint32_t* err;    // device status word (+ a few scratch words after it)
  // build / restructure scratch
  int64_t scap;
  uint64_t* keys0;
  uint64_t* keys1;
  uint32_t* vals0;
  uint32_t* vals1;
  uint32_t* hist;
  uint32_t* flags;   // [scap]
  uint32_t* flags2;  // [scap]
  uint64_t* grown;   // [nnz] accepted regrowth positions
  uint8_t* vcopy;    // [nnz * 4] copy of values
  uint32_t* scan_tmp;
};

namespace snk {

// format.cu
struct Workspace;
snk_status layout_carve(snk_layout* L, void* ws, size_t ws_bytes);
size_t workspace_bytes(int64_t M, int64_t K, int64_t nnz, int32_t P);
snk_status build_format(snk_layout* L, void* values, int vbytes, cudaStream_t s);
snk_status derive_format(snk_layout* L, cudaStream_t s);
snk_status restructure(snk_layout* L, void* values, int64_t k, uint64_t seed, float regrow_value,
                       int32_t* old_to_new, cudaStream_t s);

// spmm.cu
snk_status launch_spmm(const snk_layout* L, bool transpose, const void* values, const void* B,
                       int64_t N, int64_t ldb, void* C, int64_t ldc, cudaStream_t s);
snk_status launch_sddmm(const snk_layout* L, const void* dY, int64_t lddy, const void* X, int64_t ldx,
                        int64_t N, void* dW, cudaStream_t s);
snk_status launch_zero_rows(void* C, int64_t rows, int64_t N, int64_t ldc, int elem_bytes, cudaStream_t s);
snk_status remap_entries(const int32_t* old_to_new, int64_t nnz, const void* src, void* dst, int elem_bytes,
                         cudaStream_t s);

}  // namespace snk

#define SNK_CUDA_TRY(expr)                   \
  do {                                       \
    cudaError_t e__ = (expr);                \
    if (e__ != cudaSuccess) {                \
      (void)cudaGetLastError();              \
      return SNK_ERR_CUDA;                   \
    }                                        \
  } while (0)

#define SNK_TRY(expr)               \
  do {                              \
    snk_status s__ = (expr);        \
    if (s__ != SNK_OK) return s__;  \
  } while (0)
