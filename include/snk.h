/*
 * snk.h -- C ABI of the truly-sparse layer library (libsnk.so, CUDA, sm_100a).
 *
 * The layer follows "Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural Networks on
 * GPU" (arXiv 2610.04093), Abstract: the weight W (M x K) is stored only as its nonzero
 * connections in COO format, the forward product and both backward products run
 * "entirely in the sparse paradigm", and an API restructures the connection set.  The
 * pages name the operations but print no code or interface; the calls below are this
 * library's own design.
 *
 * Conventions shared by every call
 *  - All array arguments are DEVICE pointers on the device that was current at
 *    snk_build.  The caller owns every buffer: COO arrays, values, activations,
 *    outputs and the workspace.  The library never allocates device memory.
 *  - Dense operands are row-major with a leading dimension (elements between row
 *    starts) >= their column count.  X and dX are K x N, Y and dY are M x N.
 *  - Values and activations share one element type (snk_dtype); accumulation is fp32;
 *    each output is rounded once (round to nearest even for bf16).  Outputs are
 *    overwritten, never accumulated into.
 *  - Index arrays are int32 (nnz < 2^31, M and K < 2^31).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  snk_forward,
 *    snk_backward_input and snk_backward_weight only check arguments on the host and
 *    enqueue kernels: they never synchronise.  snk_build and snk_restructure synchronise
 *    `stream` once (or once per regrowth round) to read the device status word.
 *  - No call aborts, traps or prints.  Errors are returned as snk_status; on an error
 *    no caller array has been modified unless the call's comment says otherwise.
 */
#ifndef SNK_H
#define SNK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SNK_API __attribute__((visibility("default")))
#else
#define SNK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* snk_stream; /* identical to cudaStream_t */

typedef enum {
  SNK_OK = 0,
  SNK_ERR_INVALID_ARG = 1,          /* bad size, null pointer, dtype mismatch, ld < N ... */
  SNK_ERR_OUT_OF_RANGE = 2,         /* a COO index outside [0, M) x [0, K) */
  SNK_ERR_DUPLICATE = 3,            /* a (row, col) position given twice */
  SNK_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes < snk_workspace_bytes(...) */
  SNK_ERR_UNSUPPORTED = 5,          /* sizes beyond the int32 index range */
  SNK_ERR_INVALID_VALUE = 6,        /* a NaN value where values are ranked (restructure) */
  SNK_ERR_NO_ROOM = 7,              /* restructure: drop_count > M*K - nnz */
  SNK_ERR_TIMEOUT = 8,              /* restructure: regrowth did not finish within its bound */
  SNK_ERR_CUDA = 9                  /* a CUDA runtime call or kernel launch failed */
} snk_status;

typedef enum { SNK_F32 = 0, SNK_BF16 = 1 } snk_dtype;

/* Opaque host object describing one built layout; it points into the caller's
 * workspace and at the caller's (sorted) row/col arrays, and holds no device memory. */
typedef struct snk_layout snk_layout;

/* Read-only view of a layout's device arrays (for tests and tooling). */
typedef struct {
  int64_t M, K, nnz;
  int32_t num_parts;  /* P actually used (<= max(nnz, 1)) */
  int32_t dtype;      /* snk_dtype */
  int32_t device;
  const int32_t* row;        /* [nnz] sorted COO rows (caller's array) */
  const int32_t* col;        /* [nnz] sorted COO cols (caller's array) */
  const int32_t* row_ptr;    /* [M+1] row_ptr[r] = #entries with row < r */
  const int32_t* col_ptr;    /* [K+1] col_ptr[c] = #entries with col < c */
  const int32_t* csc_row;    /* [nnz] csc_row[j] = row[perm[j]] */
  const int32_t* perm;       /* [nnz] sorted-COO index of the j-th entry in (col, row) order */
  const int32_t* part_nnz;   /* [P+1] part_nnz[p] = floor(p * nnz / P) */
  const int32_t* part_row;   /* [P+1] row holding entry part_nnz[p]; M when it equals nnz */
  const int32_t* part_nnz_t; /* [P+1] same split over the column-ordered entries */
  const int32_t* part_col;   /* [P+1] column holding entry part_nnz_t[p]; K when it equals nnz */
} snk_layout_view;

/* Human-readable name of a status ("SNK_OK", ...).  Never NULL. */
SNK_API const char* snk_status_string(snk_status s);

/* Default number of nnz-balanced parts for `nnz` entries on a GPU with `sm_count` SMs:
 * min(3 * sm_count, ceil(nnz / 256)), at least 1 (the product kernels keep three CTAs of
 * 256 threads resident per SM, so the default is one wave).  Pure host arithmetic. */
SNK_API int32_t snk_default_num_parts(int64_t nnz, int32_t sm_count);

/* Bytes of device workspace a layout with these sizes needs (num_parts as passed to
 * snk_build; 0 = the default for the current device, which this call then queries).
 * Returns 0 for invalid sizes.  The size does not change under snk_restructure.  It
 * includes 4 bytes per nonzero for 16-bit index copies when M, K <= 65536. */
SNK_API size_t snk_workspace_bytes(int64_t M, int64_t K, int64_t nnz, int32_t num_parts);

/*
 * snk_build -- the COO format work ("COO-format" layer, arXiv 2610.04093 Abstract):
 *   1. validate 0 <= row < M and 0 <= col < K (else SNK_ERR_OUT_OF_RANGE) and reject a
 *      repeated (row, col) (SNK_ERR_DUPLICATE);
 *   2. sort the entries by (row, col) IN PLACE in `row`, `col`, `values` (values move
 *      bit-exactly with their entries);
 *   3. derive row_ptr, the CSC permutation (perm, col_ptr, csc_row) and P nnz-balanced
 *      parts over both orders (see snk_layout_view).
 * row, col: int32 [nnz], any order.  values: [nnz] of `vdt`.  workspace: device buffer
 * of ws_bytes >= snk_workspace_bytes(M, K, nnz, num_parts), 256-byte aligned, that must
 * outlive the layout.  row/col/values/workspace stay owned by the caller; the layout keeps
 * pointers to row, col and workspace (not to values).  On success *out receives a new
 * layout (free it with snk_destroy).  On any error the COO arrays are left unchanged and
 * *out is NULL.  Synchronises `stream`.
 */
SNK_API snk_status snk_build(int64_t M, int64_t K, int64_t nnz, int32_t* row, int32_t* col, void* values,
                     snk_dtype vdt, int32_t num_parts, void* workspace, size_t ws_bytes,
                     snk_stream stream, snk_layout** out);

/*
 * snk_forward -- Y = W X, Y[r, n] = sum over entries e of row r of v_e * X[col_e, n]
 * (the SpMM the Abstract of arXiv 2610.04093 measures "at the kernel level").
 * values: [nnz] in the layout's sorted order.  X: K x N (ldx >= N).  Y: M x N (ldy >= N),
 * overwritten.  dt must equal the layout's dtype.  Asynchronous on `stream`.  Uses a
 * per-layout scratch region: calls of snk_forward on one layout must not overlap in time
 * (snk_backward_input has its own region and may overlap with snk_forward).
 * For N >= 256 with X 16-byte aligned (base and ldx * element size) the product runs in the
 * tensor-copy-staged wide kernel, whose shared-memory barrier waits are bounded (a wait
 * that runs out is reported by snk_sync_status); other shapes take the nnz-balanced
 * kernel.  The same holds for snk_backward_input with dY.
 */
SNK_API snk_status snk_forward(const snk_layout* L, const void* values, const void* X, int64_t N, int64_t ldx,
                       void* Y, int64_t ldy, snk_dtype dt, snk_stream stream);

/*
 * snk_backward_input -- dX = W^T dY, dX[c, n] = sum over entries e of column c of
 * v_e * dY[row_e, n] (the input gradient of "backpropagating gradients entirely in the
 * sparse paradigm", arXiv 2610.04093 Abstract), walked through the CSC permutation.
 * dY: M x N (lddy >= N).  dX: K x N (lddx >= N), overwritten.  Asynchronous.  Calls on
 * one layout must not overlap each other in time.
 */
SNK_API snk_status snk_backward_input(const snk_layout* L, const void* values, const void* dY, int64_t N,
                              int64_t lddy, void* dX, int64_t lddx, snk_dtype dt, snk_stream stream);

/*
 * snk_backward_weight -- the sampled weight gradient (SDDMM): dW[e] = sum over n of
 * dY[row_e, n] * X[col_e, n], i.e. dY X^T read at the stored positions only (same
 * passage as above).  dY: M x N, X: K x N.  dW: [nnz] of dt in the layout's sorted
 * order, overwritten.  Asynchronous; uses no scratch, so calls may overlap freely.
 */
SNK_API snk_status snk_backward_weight(const snk_layout* L, const void* dY, int64_t lddy, const void* X,
                               int64_t ldx, int64_t N, void* dW, snk_dtype dt, snk_stream stream);

/*
 * snk_restructure -- prune and regrow connections ("a simple PyTorch API for
 * restructuring connections", arXiv 2610.04093 Abstract; Dynamic Sparse Training).
 * The pages give no rule; this library's reading:
 *   1. drop the drop_count entries of smallest |value| (bf16 widened exactly; -0 == +0),
 *      ties to the smaller linear index row*K + col; a NaN value is SNK_ERR_INVALID_VALUE;
 *   2. regrow drop_count positions: walk SplitMix64 seeded with `seed`, draw u_i maps to
 *      position floor(u_i * M*K / 2^64); accept a position not in the pre-drop set and not
 *      accepted before; stop at drop_count acceptances (SNK_ERR_NO_ROOM when
 *      drop_count > M*K - nnz; SNK_ERR_TIMEOUT if 2^32 draws do not suffice);
 *   3. regrown entries get regrow_value rounded to the value type; survivors keep their
 *      value bits;
 *   4. rewrite the layout's row/col arrays and `values` in (row, col) order and rebuild
 *      every derived array.  nnz is unchanged.
 * old_to_new: optional int32 [nnz] (device) receiving the new index of each old entry,
 * -1 for dropped ones (to remap optimizer state).  Synchronises `stream`.  Must not
 * overlap with any other call on the same layout.  On an error before the rewrite
 * (INVALID_ARG, INVALID_VALUE, NO_ROOM, TIMEOUT) nothing is modified.
 */
SNK_API snk_status snk_restructure(snk_layout* L, void* values, int64_t drop_count, uint64_t seed,
                           float regrow_value, int32_t* old_to_new, snk_stream stream);

/*
 * snk_csr_forward_static -- Y = W X straight from a CSR matrix, allocating nothing.
 * (This entry point is the library's own addition; the paper has no counterpart.)
 * For callers that cannot allocate device memory at all -- e.g. code given a CSR matrix
 * and its activation buffers by a host framework that owns every allocation -- and so
 * cannot provide the workspace that snk_build needs.  The kernel's scratch (work
 * descriptors, carry slots of rows split between CTAs and their arrival counters) lives
 * in a fixed static device array of about 0.4 MB that every GPU loading the library holds
 * until process exit; at most SNK_STATIC_MAX_PARTS CTAs use it per launch.
 * row_ptr: int32 [M+1] (row_ptr[0] = 0, non-decreasing, row_ptr[M] = nnz); col: int32
 * [nnz] in [0, K); values: [nnz] of dt.  The arrays are NOT validated: an index outside
 * its range is undefined behaviour.  X: K x N (ldx >= N); Y: M x N (ldy >= N),
 * overwritten.  num_parts: 0 = the default split, else 1..SNK_STATIC_MAX_PARTS (larger
 * values return SNK_ERR_UNSUPPORTED).  Calls no allocator.  The first call on a device
 * looks up the scratch array's device address, so make it before any stream capture on
 * that device.  Every call shares the one scratch array (counters are cleared at the
 * start of each call): calls that overlap on the GPU, on any stream, race.
 */
#define SNK_STATIC_MAX_PARTS 512
SNK_API snk_status snk_csr_forward_static(int64_t M, int64_t K, int64_t nnz, const int32_t* row_ptr,
                                          const int32_t* col, const void* values, snk_dtype dt, const void* X,
                                          int64_t N, int64_t ldx, void* Y, int64_t ldy, int32_t num_parts,
                                          snk_stream stream);

/* Fill *v with the layout's sizes and device pointers.  Returns SNK_ERR_INVALID_ARG for
 * NULL arguments. */
/*
 * snk_remap_entries -- carries per-entry state (optimizer moments, masks, ...) across a
 * snk_restructure: dst[old_to_new[e]] = src[e] for every e with old_to_new[e] >= 0, and
 * every other dst entry (the regrown connections) is set to zero.  old_to_new: the int32
 * [nnz] map snk_restructure wrote; src, dst: device [nnz] arrays of elem_bytes (2 or 4)
 * each, not aliased.  Asynchronous on `stream` (on the current device); SNK_ERR_INVALID_ARG
 * for bad sizes, null or aliased pointers.  (A library addition: the training loop of
 * dynamic sparse training needs it; the pages name the use, not the call.)
 */
SNK_API snk_status snk_remap_entries(const int32_t* old_to_new, int64_t nnz, const void* src, void* dst,
                                     int32_t elem_bytes, snk_stream stream);

/*
 * snk_set_index_bits -- the width of the column / row indices the products read: 32 (the
 * format as built, the default) or 16.  Index bytes are a cost the essay "Two Lotteries"
 * names for unstructured formats; when both M and K are <= 65536 the layout also keeps
 * 16-bit copies of col and csc_row (in the workspace, refreshed by snk_restructure), and
 * bits = 16 makes the forward, transposed and SDDMM kernels read those instead: 2 bytes
 * per nonzero less (perm stays 32-bit).  Results are bit-identical either way.  Takes
 * effect for calls made after it; SNK_ERR_INVALID_ARG for other widths,
 * SNK_ERR_UNSUPPORTED for 16 when a dimension exceeds 65536.  (A library addition.)
 */
SNK_API snk_status snk_set_index_bits(snk_layout* L, int32_t bits);

/*
 * snk_im2col3x3 -- the patch matrix of a 3x3 convolution (stride 1, zero padding 1, no
 * bias), so that a sparse 3x3 layer is snk_forward with K = 9 C on it ("SparseRT", arXiv
 * 2008.11849, Abstract: sparse 1x1 and 3x3 convolutions).  x: C x Nb x H x W, channel-major
 * and contiguous, of dt.  out: (9 C) x (Nb H W) with leading dimension ld >= Nb H W:
 * out[ci*9 + kh*3 + kw][(n*H + h)*W + w] = x[ci][n][h+kh-1][w+kw-1], or zero outside the
 * image -- the column index of a [Co][C][3][3] weight flattened row-major.  Elements are
 * copied bit for bit.  Asynchronous on `stream` (current device).  SNK_ERR_INVALID_ARG for
 * sizes <= 0, 9 C > 65535, ld < Nb H W, null pointers or another dtype.  (The explicit
 * patch matrix costs 9x the input in HBM traffic; the convolution oracle is the plain
 * definition.)
 */
SNK_API snk_status snk_im2col3x3(const void* x, int64_t C, int64_t Nb, int64_t H, int64_t W, void* out, int64_t ld,
                                 snk_dtype dt, snk_stream stream);

/*
 * snk_sync_status -- synchronises `stream` and reports whether a product launch on this
 * layout gave up a bounded wait: the TMA-staged kernels for wide operands wait on
 * shared-memory barriers for the tensor copies, each wait for at most about a second.
 * Returns SNK_ERR_TIMEOUT then (and clears the layout's status word), SNK_OK otherwise.
 * The products never synchronise; this is how a caller that wants to know checks.
 * (A library addition; the paper has no counterpart.)
 */
SNK_API snk_status snk_sync_status(snk_layout* L, snk_stream stream);

/*
 * snk_probe_fp32_fma -- a measurement aid, not part of the method: launches `blocks` CTAs
 * of chains of packed fp32 FMAs, `iters` steps each, on `stream`, so that a caller timing
 * it with events learns the GPU's fp32 FMA rate (the ALU roofline of the products when
 * N is large).  snk_probe_fp32_fma_flops returns the floating-point operations of such a
 * launch (an FMA counts 2).  sink: device float [blocks], normally left unwritten.
 * Asynchronous; SNK_ERR_INVALID_ARG for blocks or iters <= 0 or a NULL sink.
 */
SNK_API snk_status snk_probe_fp32_fma(int32_t blocks, int32_t iters, float* sink, snk_stream stream);
SNK_API int64_t snk_probe_fp32_fma_flops(int32_t blocks, int32_t iters);

SNK_API snk_status snk_layout_info(const snk_layout* L, snk_layout_view* v);

/* Free the host object (no device memory is freed; the caller owns the workspace). */
SNK_API void snk_destroy(snk_layout* L);

#ifdef __cplusplus
}
#endif

#endif /* SNK_H */
