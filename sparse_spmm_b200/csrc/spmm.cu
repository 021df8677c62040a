// spmm.cu -- the three products of the truly-sparse layer on CUDA cores (sm_100a):
//   forward      Y  = W X      (CSR walk over the row-sorted COO)
//   transposed   dX = W^T dY   (the same kernel walking the CSC permutation)
//   SDDMM        dW = (dY X^T) read at the stored positions
// ("Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural Networks on GPU",
// arXiv 2610.04093, Abstract: forward and sparse backpropagation of a COO layer).
//
// Work split (the load-balance argument of "Two Lotteries: What It Takes to Make
// Sparsity Fast", section on uneven work: a fixed per-unit assignment lets the busiest
// unit set the time): the nnz are cut into P equal parts, one CTA per part, whatever
// the row lengths; a precomputed descriptor moves each part's ends to row boundaries
// unless the row there is longer than a part.  Inside a CTA the range is cut again into
// equal contiguous pieces, one per "worker" (G lanes that share one entry stream and
// split the dense columns, NC per lane).  A worker walks its piece in order with a
// running fp32 sum per row; rows that complete inside the worker are written directly.
// Partial rows at worker edges are combined by a segmented scan across the CTA's
// workers, and partial rows at CTA edges (long rows only) by fp32 carry slots: every CTA
// holding part of such a row writes its partial and bumps that row's arrival counter;
// the last one to arrive sums the partials in part order and writes the row (no waiting,
// deterministic order).  Outputs are rounded once.  No tensor cores: the gather is not a
// dense contraction.
//
// Gathered rows of the dense operand are kept packed (bf16 pairs in 32-bit words) until
// the FMA and are multiplied with packed fp32 FMAs (two lanes of fp32 per instruction).
// A lane holds up to 32 bytes of a row (one 32-byte load where aligned), so few lanes
// repeat the per-entry index and value loads.  Before waiting on the previous grid the
// CTAs prefetch their share of every operand into L2.
//
// Wide dense operands (N >= 256) take a different kernel, k_spmm_tma: row blocks x
// 128-column slices, the dense operand staged through shared memory by tensor-memory
// copies in a warp-specialised producer/consumer pipeline (see its own comment).
#include <algorithm>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "internal.cuh"

namespace snk {
namespace {

constexpr int kThreads = 256;
constexpr int kRowCap = 2048;   // row_ptr slice entries held in shared memory per CTA
constexpr int kStageCap = 4096; // SDDMM results staged in shared memory per CTA
constexpr unsigned kFull = 0xffffffffu;

__host__ __device__ __forceinline__ int64_t mn64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------------------- element I/O

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float load1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) {
  return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ void store1(float* p, float v) { *p = v; }
__device__ __forceinline__ void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// NC consecutive elements of T held as loaded: 32-bit words (two bf16 per word, or one
// float).  Groups of more than one element are loaded with aligned vector loads of up to
// 16 bytes each (the host guarantees 16-byte alignment of every row start and column).
template <typename T, int NC>
struct Packed {
  static constexpr int W = sizeof(T) == 2 ? (NC + 1) / 2 : NC;
  uint32_t w[W];
};

template <int NC, typename T>
__device__ __forceinline__ void load_packed(const T* p, Packed<T, NC>& r, bool a32 = false) {
  constexpr int W = Packed<T, NC>::W;
  if constexpr (W == 8) {
    if (a32) {  // one 32-byte load
      asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                   : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]),
                     "=r"(r.w[6]), "=r"(r.w[7])
                   : "l"(p));
      return;
    }
  }
  if constexpr (W >= 4) {
#pragma unroll
    for (int k = 0; k < W; k += 4) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + k / 4);
      r.w[k] = v.x; r.w[k + 1] = v.y; r.w[k + 2] = v.z; r.w[k + 3] = v.w;
    }
  } else if constexpr (W == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    r.w[0] = v.x; r.w[1] = v.y;
  } else if constexpr (sizeof(T) == 2 && NC == 1) {
    r.w[0] = (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16;  // one value, high half
  } else {
    r.w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
  }
}

template <typename T, int NC>
__device__ __forceinline__ void zero_packed(Packed<T, NC>& r) {
#pragma unroll
  for (int k = 0; k < Packed<T, NC>::W; ++k) r.w[k] = 0u;
}

// Unpacked value j of a packed group.
template <typename T, int NC>
__device__ __forceinline__ float unpack(const Packed<T, NC>& r, int j) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (NC == 1) return __uint_as_float(r.w[0]);
    return (j & 1) ? bf_hi(r.w[j >> 1]) : bf_lo(r.w[j >> 1]);
  } else {
    return __uint_as_float(r.w[j]);
  }
}

// NC fp32 accumulators held as register pairs, so packed FMAs need no repacking.
template <int NC>
struct Acc {
  float2 p[(NC + 1) / 2];
  __device__ __forceinline__ float& operator[](int j) { return (j & 1) ? p[j >> 1].y : p[j >> 1].x; }
  __device__ __forceinline__ float operator[](int j) const { return (j & 1) ? p[j >> 1].y : p[j >> 1].x; }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int k = 0; k < (NC + 1) / 2; ++k) p[k] = make_float2(0.f, 0.f);
  }
};

// acc[j] += v * x[j] for the NC columns, two columns per packed fp32 FMA.
template <typename T, int NC>
__device__ __forceinline__ void fma_row(float v, const Packed<T, NC>& x, Acc<NC>& acc) {
  if constexpr (NC == 1) {
    acc.p[0].x = fmaf(v, unpack<T, NC>(x, 0), acc.p[0].x);
  } else {
    const float2 vv = make_float2(v, v);
#pragma unroll
    for (int j = 0; j < NC; j += 2)
      acc.p[j / 2] = __ffma2_rn(vv, make_float2(unpack<T, NC>(x, j), unpack<T, NC>(x, j + 1)), acc.p[j / 2]);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Store NC values (rounded once to T) with aligned vector stores of up to 16 bytes.
template <int NC, typename T>
__device__ __forceinline__ void store_cols(T* p, const float* v) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (NC >= 8) {
#pragma unroll
      for (int k = 0; k < NC; k += 8)
        reinterpret_cast<uint4*>(p)[k / 8] = make_uint4(pack_bf16x2(v[k], v[k + 1]), pack_bf16x2(v[k + 2], v[k + 3]),
                                                        pack_bf16x2(v[k + 4], v[k + 5]), pack_bf16x2(v[k + 6], v[k + 7]));
    } else if constexpr (NC == 4) {
      *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else if constexpr (NC == 2) {
      *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(v[0], v[1]);
    } else {
      store1(p, v[0]);
    }
  } else {
    if constexpr (NC >= 4) {
#pragma unroll
      for (int k = 0; k < NC; k += 4)
        reinterpret_cast<float4*>(p)[k / 4] = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
    } else if constexpr (NC == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
      p[0] = v[0];
    }
  }
}

template <int NC, typename T>
__device__ __forceinline__ void store_cols(T* p, const Acc<NC>& a) {
  float v[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) v[j] = a[j];
  store_cols<NC>(p, v);
}

template <int NC, typename T>
__device__ __forceinline__ void store_zero(T* p) {
  float z[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) z[j] = 0.f;
  store_cols<NC>(p, z);
}

// ------------------------------------------------------------------------- launch ordering

// Programmatic dependent launch: every product kernel lets the next kernel in the stream
// start launching at once, and waits for the previous grid (and its memory) before it
// touches global memory, since any input may have been written by that grid.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bulk L2 prefetch of the 16-byte-aligned bytes inside [p, p + bytes).  Only a hint: L2 is
// the point of coherence, so it may run before the previous grid has finished writing.
__device__ __forceinline__ void prefetch_l2(const void* p, int64_t bytes) {
  const uintptr_t lo = ((uintptr_t)p + 15) & ~(uintptr_t)15;
  const uintptr_t hi = ((uintptr_t)p + (uintptr_t)bytes) & ~(uintptr_t)15;
  if (bytes > 0 && hi > lo && hi - lo < (1u << 30))
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo), "r"((uint32_t)(hi - lo)) : "memory");
}

// Slice part of P of an array of n elements of E bytes: [n * part / P, n * (part + 1) / P).
template <int E>
__device__ __forceinline__ void prefetch_slice(const void* base, int64_t n, int part, int P) {
  const int64_t i0 = n * part / P, i1 = n * (part + 1) / P;
  prefetch_l2(static_cast<const char*>(base) + i0 * E, (i1 - i0) * E);
}

// f(integral_constant<int, I>) for I = B .. E-1, unrolled at compile time.
template <int B, int E, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>{});
    static_for<B + 1, E>(f);
  }
}

// Last r in [lo, hi] with rp(r) <= x.
template <typename RPF>
__device__ __forceinline__ int64_t search_row(RPF rp, int64_t lo, int64_t hi, int64_t x) {
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (rp(mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------------- SpMM (fwd / transposed)

template <typename T, typename I>
struct SpmmArgs {
  const int32_t* ptr;  // [rows + 1] row_ptr (forward) or col_ptr (transposed)
  const I* idx;        // [nnz] col (forward) or csc_row (transposed), 32- or 16-bit
  const int32_t* perm; // [nnz] transposed only: sorted-COO index of the j-th CSC entry
  const T* vals;       // [nnz] values in sorted-COO order
  const int4* desc;    // [P] per-CTA work descriptors {a, b, ra, rb}
  const T* B;          // gathered dense operand (X or dY), offset to this launch's columns
  T* C;                // output (Y or dX), offset to this launch's columns
  int64_t ldb, ldc;
  int64_t rows;        // output rows
  int64_t nnz;
  int P;
  int ncols;           // columns in this launch (<= kCarryCols, a multiple of NC)
  int b32;             // every gathered row offset c * ldb fits in 32 bits
  int a32;             // every gathered lane group is 32-byte aligned
  int64_t bbytes;      // bytes of the gathered operand when it is one dense block, else 0
  int64_t prows;       // entries of ptr
  float* carry_tail;   // [P][kCarryCols]
  float* carry_head;   // [P][kCarryCols]
  uint32_t* cnt;       // [kMaxTiles][P], zero between launches
};

// Transposed, with 16- or 32-byte lane groups, the value positions are loaded one batch ahead
// of the values (the batches are long enough for the second stage to pay).
template <typename T, int NC, bool TRANS>
constexpr bool perm_ahead() { return TRANS && NC * (int)sizeof(T) >= 16; }
// Entries in flight per worker: as many as the register budget of 3 CTAs per SM allows.
template <typename T, int NC, bool TRANS = false>
constexpr int spmm_batch() {
  return NC * (int)sizeof(T) >= 32 ? 3 : (NC * (int)sizeof(T) >= 16 ? (perm_ahead<T, NC, TRANS>() ? 5 : 6) : 8);
}
// SDDMM entries in flight per worker.  DEEP (wide operands, several column passes per entry)
// measured best with more entries in flight, short operands with fewer (registers).
template <typename T, int NC, bool DEEP = false>
constexpr int sddmm_batch() {
  return NC * (int)sizeof(T) >= 32 ? (DEEP ? 4 : 3) : (NC * (int)sizeof(T) >= 8 ? 4 : 6);
}

template <typename T, int NC, int G, bool TRANS, typename I>
__global__ void __launch_bounds__(kThreads, 3) k_spmm_small(const SpmmArgs<T, I> A) {
  constexpr int NW = kThreads / G;   // workers per CTA
  constexpr int WPW = 32 / G;        // workers per warp
  constexpr int NT = NC * G;         // columns per tile
  constexpr int NWARPS = kThreads / 32;
  constexpr int UB = spmm_batch<T, NC, TRANS>();
  constexpr bool PA = perm_ahead<T, NC, TRANS>();
  __shared__ int32_t s_rp[kRowCap];
  __shared__ float s_agg[NWARPS][NT];
  __shared__ int s_aggF[NWARPS];
  __shared__ float s_head[NC][kThreads];  // the worker's first, still open row (per lane)

  pdl_launch_dependents();
  const int part = blockIdx.x, tile = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int w = tid / G, l = tid % G, g = lane / G;
  const int lane_base = lane - l;
  const unsigned gmask = G == 32 ? kFull : (((1u << G) - 1u) << lane_base);
  const int n0 = tile * NT + l * NC;
  const bool active = n0 < A.ncols;  // this lane holds NC real columns (or none)
  if (tile == 0 && lane == 0) {
    // L2 warm-up while the previous grid drains: together the CTAs cover every operand once.
    if (wp == 0) {
      prefetch_l2(A.desc + part, sizeof(int4));
      prefetch_slice<4>(A.ptr, A.prows, part, A.P);
    } else if (wp == 1) {
      prefetch_slice<sizeof(I)>(A.idx, A.nnz, part, A.P);
    } else if (wp == 2) {
      prefetch_slice<sizeof(T)>(A.vals, A.nnz, part, A.P);
    } else if (wp == 3) {
      if (TRANS) prefetch_slice<4>(A.perm, A.nnz, part, A.P);
    } else if (wp == 4) {
      prefetch_slice<1>(A.B, A.bbytes, part, A.P);
    }
  }
  pdl_wait();

  const int4 dsc = __ldg(A.desc + part);
  const int64_t a = dsc.x, b = dsc.y, ra = dsc.z, rb = dsc.w;
  const int np = (int)(b - a);
  // the worker's piece, as offsets from a
  const int s = (int)(((int64_t)np * w) / NW);
  const int e_end = (int)(((int64_t)np * (w + 1)) / NW);
  const I* __restrict__ idx = A.idx + a;
  const int32_t* __restrict__ prm = TRANS ? A.perm + a : nullptr;
  const T* __restrict__ vals = TRANS ? A.vals : A.vals + a;

  // the worker's next batch of indices / values (prefetched one batch ahead); with PA the
  // value positions run one batch further ahead, so each value gather waits on one load only
  int c[UB];
  float v[UB];
  int pn[PA ? UB : 1];
  auto load_perm = [&](int e0, int nb) {
    if constexpr (PA) {
#pragma unroll
      for (int i = 0; i < UB; ++i)
        if (i < nb) pn[i] = __ldg(prm + e0 + i);
    }
  };
  auto load_batch = [&](int e0, int nb) {
#pragma unroll
    for (int i = 0; i < UB; ++i) {
      if (i < nb) {
        c[i] = __ldg(idx + e0 + i);
        if constexpr (PA) v[i] = load1(vals + pn[i]);
        else v[i] = TRANS ? load1(vals + __ldg(prm + e0 + i)) : load1(vals + e0 + i);
      }
    }
    const int e1 = e0 + nb;  // the batch after this one
    if (PA && e1 < e_end) load_perm(e1, min(UB, e_end - e1));
  };
  if (s < e_end) {
    load_perm(s, min(UB, e_end - s));
    load_batch(s, min(UB, e_end - s));
  }

  const int64_t rhi = mn64(rb + 1, A.rows);
  const int64_t span = rhi - ra + 1;
  const bool in_smem = np > 0 && span <= kRowCap;
  if (in_smem)
    for (int64_t i = tid; i < span; i += kThreads) s_rp[i] = __ldg(A.ptr + ra + i);
  __syncthreads();
  // row pointers, relative to a
  auto RP = [&](int64_t r) -> int { return (in_smem ? s_rp[r - ra] : __ldg(A.ptr + r)) - (int)a; };

  const T* __restrict__ Bb = A.B + n0;
  T* __restrict__ Cb = A.C + n0;
  const unsigned ldb = (unsigned)A.ldb;
  const bool small_b = A.b32 != 0;
  const bool a32 = A.a32 != 0;

  Acc<NC> acc;
  acc.zero();
  bool has_head = false, has_tail = false, link = true;
  int64_t h_row = -1;

  if (s < e_end) {
    int64_t r = search_row([&](int64_t q) { return (int64_t)RP(q); }, ra, mn64(rb, A.rows - 1), s);
    int r_end = RP(r + 1);
    bool first = true, open = RP(r) < s;
    if (s == 0 && a == 0 && active)  // empty rows ahead of the first entry
      for (int64_t q = 0; q < r; ++q) store_zero<NC>(Cb + q * A.ldc);

    auto finish = [&](int64_t row) {
      if (first && open) {
        has_head = true;
        h_row = row;
#pragma unroll
        for (int j = 0; j < NC; ++j) s_head[j][tid] = acc[j];
      } else if (active) {
        store_cols<NC>(Cb + row * A.ldc, acc);
      }
      first = false;
      open = false;
      acc.zero();
    };

    int e = s;
    while (e < e_end) {
      const int nb = min(UB, e_end - e);
      Packed<T, NC> x[UB];
      float vv[UB];
#pragma unroll
      for (int i = 0; i < UB; ++i) {
        vv[i] = v[i];
        if (i < nb && active) {
          const T* src = small_b ? Bb + (unsigned)c[i] * ldb : Bb + (int64_t)c[i] * A.ldb;
          load_packed<NC>(src, x[i], a32);
        } else {
          zero_packed(x[i]);
        }
      }
      const int en = e + nb;
      if (en < e_end) load_batch(en, min(UB, e_end - en));
      if (en <= r_end) {  // the whole batch lies inside row r
#pragma unroll
        for (int i = 0; i < UB; ++i)
          if (i < nb) fma_row(vv[i], x[i], acc);
      } else {
#pragma unroll
        for (int i = 0; i < UB; ++i) {
          if (i < nb) {
            while (e + i >= r_end) {
              finish(r);
              ++r;
              r_end = RP(r + 1);
            }
            fma_row(vv[i], x[i], acc);
          }
        }
      }
      e = en;
    }
    if (r_end == e_end) {
      finish(r);
      link = false;
      while (r + 1 < A.rows && RP(r + 2) == e_end) {  // empty rows right after this range
        ++r;
        if (active) store_zero<NC>(Cb + r * A.ldc);
      }
    } else {
      has_tail = true;       // acc holds the open row's partial
      link = first && open;  // the whole range lies inside one row that started earlier
    }
  }

  // Segmented inclusive scan of the workers' tail partials (segments = rows); acc becomes
  // the scanned value S.
#pragma unroll
  for (int j = 0; j < NC; ++j) acc[j] = has_tail ? acc[j] : 0.f;
  int F = link ? 0 : 1;
#pragma unroll
  for (int off = 1; off < WPW; off <<= 1) {
    const int Fp = __shfl_up_sync(kFull, F, off * G);
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const float sp = __shfl_up_sync(kFull, acc[j], off * G);
      if (g >= off && !F) acc[j] += sp;
    }
    if (g >= off) F |= Fp;
  }
  if (g == WPW - 1) {
#pragma unroll
    for (int j = 0; j < NC; ++j) s_agg[wp][l * NC + j] = acc[j];
    if (l == 0) s_aggF[wp] = F;
  }
  __syncthreads();
  // warp 0 turns the warp aggregates into their segmented exclusive prefix, one column per
  // lane (measured 2-3% faster than every warp folding the aggregates before it)
  if (wp == 0) {
    for (int c = lane; c < NT; c += 32) {
      float h = 0.f;
      for (int q = 0; q < NWARPS; ++q) {
        const float a = s_agg[q][c];
        s_agg[q][c] = h;
        h = s_aggF[q] ? a : h + a;
      }
    }
  }
  __syncthreads();
  float H[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) H[j] = s_agg[wp][l * NC + j];  // the incoming prefix until it is added
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    const float inc = H[j];
    if (!F) acc[j] += inc;
    float ej = __shfl_up_sync(kFull, acc[j], G);  // S of the previous worker
    if (g == 0) ej = inc;
    H[j] = has_head ? s_head[j][tid] + ej : 0.f;
  }

  // Rows split across CTAs (only rows longer than a part): write this CTA's partial; the
  // last CTA to arrive sums all partials in part order and writes the row.
  auto cross_cta = [&](int64_t row, const float* val, bool row_ends_here) {
    const int64_t rs = (int64_t)RP(row) + a, re = (int64_t)RP(row + 1) + a;
    const int64_t P = A.P, nnz = A.nnz;
    const int64_t p1 = ((rs + 1) * P - 1) / nnz;  // part holding the row's first entry
    const int64_t pk = (re * P - 1) / nnz;        // part holding its last entry
    float* slot = (row_ends_here ? A.carry_head : A.carry_tail) + (int64_t)part * kCarryCols + n0;
    if (active) {
#pragma unroll
      for (int j = 0; j < NC; ++j) slot[j] = val[j];
    }
    __threadfence();
    __syncwarp(gmask);
    uint32_t* ctr = A.cnt + (int64_t)tile * P + p1;
    uint32_t old = 0;
    if (l == 0) old = atomicAdd(ctr, 1u);
    old = __shfl_sync(gmask, old, lane_base);
    if ((int64_t)old == pk - p1) {
      __threadfence();
      float sum[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) sum[j] = 0.f;
      if (active) {
        for (int64_t q = p1; q < pk; ++q) {
          const float* src = A.carry_tail + q * kCarryCols + n0;
#pragma unroll
          for (int j = 0; j < NC; ++j) sum[j] += __ldcg(src + j);
        }
        const float* src = A.carry_head + pk * kCarryCols + n0;
#pragma unroll
        for (int j = 0; j < NC; ++j) sum[j] += __ldcg(src + j);
        store_cols<NC>(Cb + row * A.ldc, sum);
      }
      if (l == 0) atomicExch(ctr, 0u);
    }
  };

  if (has_head) {
    if (h_row == ra && RP(ra) < 0)
      cross_cta(h_row, H, true);
    else if (active)
      store_cols<NC>(Cb + h_row * A.ldc, H);
  }
  if (w == NW - 1 && np > 0) {
    const int64_t t = search_row([&](int64_t q) { return (int64_t)RP(q); }, ra, mn64(rb, A.rows - 1), np - 1);
    if (RP(t + 1) > np) {
      float tv[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) tv[j] = acc[j];
      cross_cta(t, tv, false);
    }
  }
}

// ------------------------------------------------------------------------- SDDMM

template <typename T, typename I>
struct SddmmArgs {
  const int32_t* row_ptr;
  const I* col;      // [nnz], 32- or 16-bit
  const int4* desc;  // [P] per-CTA work descriptors (forward ones)
  const T* X;        // K x N
  const T* dY;       // M x N
  T* dW;             // [nnz]
  int64_t ldx, lddy;
  int64_t rows;
  int64_t nnz;
  int N;             // a multiple of NC
  int a32;           // X and dY lane groups are 32-byte aligned
  int64_t xbytes, dybytes;  // bytes of X and dY when each is one dense block, else 0
};

template <typename T, int NC>
__device__ __forceinline__ float dot_packed(const Packed<T, NC>& x, const Packed<T, NC>& y, float d) {
  if constexpr (NC == 1) {
    return fmaf(unpack<T, NC>(x, 0), unpack<T, NC>(y, 0), d);
  } else {
    float2 d2 = make_float2(d, 0.f);
#pragma unroll
    for (int j = 0; j < NC; j += 2)
      d2 = __ffma2_rn(make_float2(unpack<T, NC>(x, j), unpack<T, NC>(x, j + 1)),
                      make_float2(unpack<T, NC>(y, j), unpack<T, NC>(y, j + 1)), d2);
    return d2.x + d2.y;
  }
}

template <typename T, int NC, int G, typename I, bool DEEP>
__global__ void __launch_bounds__(kThreads, 3) k_sddmm_small(const SddmmArgs<T, I> A) {
  constexpr int NW = kThreads / G;
  constexpr int NT = NC * G;
  constexpr int UB = sddmm_batch<T, NC, DEEP>();
  __shared__ int32_t s_rp[kRowCap];
  __shared__ float s_dw[kStageCap];

  pdl_launch_dependents();
  const int part = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int w = tid / G, l = tid % G;
  const int lane_base = lane - l;
  const unsigned gmask = G == 32 ? kFull : (((1u << G) - 1u) << lane_base);
  if (lane == 0) {
    // L2 warm-up while the previous grid drains: together the CTAs cover every operand once.
    const int wp = tid >> 5, P = (int)gridDim.x;
    if (wp == 0) {
      prefetch_l2(A.desc + part, sizeof(int4));
      prefetch_slice<4>(A.row_ptr, A.rows + 1, part, P);
    } else if (wp == 1) {
      prefetch_slice<sizeof(I)>(A.col, A.nnz, part, P);
    } else if (wp == 2) {
      prefetch_slice<1>(A.X, A.xbytes, part, P);
    } else if (wp == 3) {
      prefetch_slice<1>(A.dY, A.dybytes, part, P);
    }
  }
  pdl_wait();

  const int4 dsc = __ldg(A.desc + part);
  const int64_t a = dsc.x, b = dsc.y, ra = dsc.z, rb = dsc.w;
  const int np = (int)(b - a);
  const bool staged = np <= kStageCap;
  const int s = (int)(((int64_t)np * w) / NW);
  const int e_end = (int)(((int64_t)np * (w + 1)) / NW);
  const I* __restrict__ col = A.col + a;
  int c[UB];
  auto load_batch = [&](int e0, int nb) {
#pragma unroll
    for (int i = 0; i < UB; ++i)
      if (i < nb) c[i] = __ldg(col + e0 + i);
  };
  if (s < e_end) load_batch(s, min(UB, e_end - s));
  const bool a32 = A.a32 != 0;
  const int64_t rhi = mn64(rb + 1, A.rows);
  const int64_t span = rhi - ra + 1;
  const bool in_smem = np > 0 && span <= kRowCap;
  if (in_smem)
    for (int64_t i = tid; i < span; i += kThreads) s_rp[i] = __ldg(A.row_ptr + ra + i);
  __syncthreads();
  auto RP = [&](int64_t r) -> int { return (in_smem ? s_rp[r - ra] : __ldg(A.row_ptr + r)) - (int)a; };

  if (s < e_end) {
    int64_t r = search_row([&](int64_t q) { return (int64_t)RP(q); }, ra, mn64(rb, A.rows - 1), s);
    int r_end = RP(r + 1);
    for (int e = s; e < e_end; e += UB) {
      const int nb = min(UB, e_end - e);
      int cc[UB];
      int rr[UB];
      const bool one_row = e + nb <= r_end;  // the whole batch lies inside row r
#pragma unroll
      for (int i = 0; i < UB; ++i) {
        cc[i] = c[i];
        rr[i] = (int)r;
        if (!one_row && i < nb) {
          while (e + i >= r_end) {
            ++r;
            r_end = RP(r + 1);
          }
          rr[i] = (int)r;
        }
      }
      const int en = e + nb;
      if (en < e_end) load_batch(en, min(UB, e_end - en));
      float d[UB];
#pragma unroll
      for (int i = 0; i < UB; ++i) d[i] = 0.f;
      for (int n0 = l * NC; n0 < A.N; n0 += NT) {
        Packed<T, NC> xv[UB];
#pragma unroll
        for (int i = 0; i < UB; ++i)
          if (i < nb) load_packed<NC>(A.X + (int64_t)cc[i] * A.ldx + n0, xv[i], a32);
        if (one_row) {
          Packed<T, NC> yv;
          load_packed<NC>(A.dY + (int64_t)rr[0] * A.lddy + n0, yv, a32);
#pragma unroll
          for (int i = 0; i < UB; ++i)
            if (i < nb) d[i] = dot_packed(xv[i], yv, d[i]);
        } else {
#pragma unroll
          for (int i = 0; i < UB; ++i) {
            if (i < nb) {
              Packed<T, NC> yv;
              load_packed<NC>(A.dY + (int64_t)rr[i] * A.lddy + n0, yv, a32);
              d[i] = dot_packed(xv[i], yv, d[i]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < UB; ++i) {
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) d[i] += __shfl_xor_sync(gmask, d[i], off);
      }
      if (l == 0) {
#pragma unroll
        for (int i = 0; i < UB; ++i) {
          if (i < nb) {
            if (staged) s_dw[e + i] = d[i];
            else store1(A.dW + a + e + i, d[i]);
          }
        }
      }
    }
  }
  if (staged) {  // coalesced write-out of the CTA's range
    __syncthreads();
    for (int i = tid; i < np; i += kThreads) store1(A.dW + a + i, s_dw[i]);
  }
}

// ------------------------------------------------------------------------- SpMM, wide N

// For wide dense operands the work splits over (row block, column slice) pairs instead of
// nnz parts: each CTA owns whole output rows, so no row is ever split, and row skew is
// amortised by the many column slices.  The dense operand's slice is staged through shared
// memory in chunks of dense rows, so every staged element serves all rows of the block that
// hold its column.  Every lane owns four columns (kWideCols = 128 per slice).  The bound is
// the shared-memory read of one operand element per FMA.
constexpr int kWideCols = 128;  // columns per slice (4 per lane)

template <typename T, typename I>
struct WideArgs {
  const int32_t* ptr;   // [rows + 1]
  const I* idx;         // [nnz], sorted within each row, 32- or 16-bit
  const int32_t* perm;  // transposed only
  const T* vals;
  const T* B;           // brows x N, leading dimension ldb (16-byte aligned rows)
  T* C;                 // rows x N, leading dimension ldc
  int64_t ldb, ldc;
  int64_t rows, brows;
  int N;
  uint32_t* err;        // status word (may be null): ERRBIT_TIMEOUT if a pipeline wait gave up
  uint32_t extra_tx;    // 0; a test sets it (environment) so that no chunk ever completes
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ float4 lds128(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

// ------------------------------------------------------------------------- SpMM, wide N, TMA-staged

// The row-block x column-slice kernel, as a warp-specialised pipeline.  One
// producer warp brings the dense operand's chunks (KC rows x kWideCols columns) into a
// kTmaStages-deep shared-memory ring with 2-D bulk tensor copies (TMA); completion is
// counted on a "full" mbarrier per stage.  Eight consumer warps each own RW rows of the
// row block and walk every chunk: per row, the entries that fall into the chunk are a
// prefix of the row's current 32-entry batch (found by a ballot), each broadcast from
// shared memory as {v, dense-row byte offset} so that a lane needs one 8-byte read, one
// dense-row read and two packed FMAs per entry.  A consumer warp releases a stage by
// arriving on its "empty" mbarrier; the producer refills a stage once all eight have
// released it, so no CTA-wide barrier sits in the loop and warps drift up to the ring
// depth apart.  Every wait is bounded (about a second by the global timer); one that gives
// up sets ERRBIT_TIMEOUT in the status word, all roles stop, the producer lets its issued
// copies land (again bounded), and the CTA returns.
constexpr int kTmaStages = 2;
constexpr int kTmaMinN = 256;     // narrower operands take 64-column passes of the small kernel
constexpr int kTmaConsumers = 8;  // compute warps; one more warp produces
constexpr int kTmaThreads = 32 * (kTmaConsumers + 1);

// Bytes of one broadcast entry in shared memory: 8 = {v, offset}, or 16 = {v, v, offset, 0}
// (the value pair ready for the packed FMA, no move per entry).  8 measured 10-20% faster:
// the space it frees goes to longer chunks.
constexpr int kTmaEntryBytes = 8;

// Dense rows per staged chunk: the most (a multiple of 8, at most 256) that let two CTAs --
// ring, entry buffers, barriers and the 1 KB the runtime reserves per CTA -- share one SM's
// 228 KB.  Two stages of long chunks measured faster than three of short ones: the
// per-(row, chunk) costs (ballot, tail) fall with more entries per chunk, and one chunk in
// flight covers the copy latency.
template <typename T, int RW>
constexpr int tma_kc() {
  constexpr int kPerCta = 233472 / 2 - 1024;  // bytes of shared memory for each of two CTAs
  constexpr int stat = 8 * RW * 32 * kTmaEntryBytes + 8 * RW * 8 + 64;
  constexpr int kc = (kPerCta - stat - 128) / (2 * 128 * (int)sizeof(T)) / 8 * 8;
  return kc > 256 ? 256 : kc;
}

__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase with the given parity to complete; false after about `limit_ns`.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t a, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}
[[maybe_unused]] __device__ __forceinline__ uint4 lds128u(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
[[maybe_unused]] __device__ __forceinline__ void sts128u(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

template <typename T, bool TRANS, int RW, typename I>
__global__ void __launch_bounds__(kTmaThreads, 2)
    k_spmm_tma(const WideArgs<T, I> A, const __grid_constant__ CUtensorMap tmB) {
  constexpr int E = (int)sizeof(T);
  constexpr int KC = tma_kc<T, RW>();
  constexpr int ROWB = kWideCols * E;  // bytes of one staged dense row
  constexpr int CHUNK = KC * ROWB;     // bytes of one staged chunk (the TMA box)
  extern __shared__ __align__(16) unsigned char s_tx[];  // [kTmaStages][CHUNK] from a 128-byte boundary
  __shared__ __align__(16) unsigned char s_ent[kTmaConsumers][RW][32][kTmaEntryBytes];
  __shared__ int2 s_span[kTmaConsumers][RW];  // per row: {first entry of the current batch, row end}
  __shared__ __align__(8) uint64_t s_full[kTmaStages];
  __shared__ __align__(8) uint64_t s_empty[kTmaStages];
  __shared__ volatile int s_abort;

  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * (kTmaConsumers * RW);
  const int n0 = blockIdx.y * kWideCols;
  const int ncols = min(kWideCols, A.N - n0);
  const uint32_t full0 = smem_addr(&s_full[0]), empty0 = smem_addr(&s_empty[0]);
  const uint32_t xs = (smem_addr(s_tx) + 127u) & ~127u;
  if (tid == 0) {
    for (int st = 0; st < kTmaStages; ++st) {
      mbar_init(full0 + 8 * st, 1);
      mbar_init(empty0 + 8 * st, kTmaConsumers);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_abort = 0;
  }
  __syncthreads();
  pdl_wait();  // the dense operand may come from the previous grid

  const int64_t nchunks = (A.brows + KC - 1) / KC;
  const uint64_t limit_ns = 1000000000ull;
  int64_t issued = 0;  // producer lane: chunks whose copies were issued

  float2 acc[RW][2];
  if (wp == kTmaConsumers) {
    // ---- producer
    if (lane == 0) {
      for (; issued < nchunks; ++issued) {
        const int st = (int)(issued % kTmaStages);
        if (issued >= kTmaStages &&
            !mbar_wait_bounded(empty0 + 8 * st, (uint32_t)(((issued / kTmaStages) - 1) & 1), limit_ns)) {
          s_abort = 1;
          break;
        }
        if (s_abort) break;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(full0 + 8 * st, (uint32_t)CHUNK + A.extra_tx);
        tma_load_2d(xs + st * CHUNK, &tmB, n0, (int)(issued * KC), full0 + 8 * st);
      }
    }
  } else {
    // ---- consumers: rows r0 + wp*RW + i, i < RW
    int k[RW], cl[RW];
    auto load_entry = [&](int first, int last, int& cc, uint4& ent) {
      const int j = first + lane;
      cc = 0x7fffffff;
      ent = make_uint4(0u, 0u, 0u, 0u);
      if (j < last) {
        cc = __ldg(A.idx + j);
        const float v = load1(A.vals + (TRANS ? (int64_t)__ldg(A.perm + j) : (int64_t)j));
        ent = make_uint4(__float_as_uint(v), __float_as_uint(v), (uint32_t)cc * (uint32_t)ROWB, 0u);
      }
    };
    auto prefetch_next = [&](int first, int last) {  // the batch after this one, into L1
      const int j = first + 32 + lane;
      if (j < last) {
        asm volatile("prefetch.global.L1 [%0];" ::"l"(A.idx + j));
        if (TRANS) asm volatile("prefetch.global.L1 [%0];" ::"l"(A.perm + j));
      }
    };
    const uint32_t ent0 = smem_addr(&s_ent[wp][0][0][0]);
    auto ent_store = [&](uint32_t a, const uint4& e) {
      if constexpr (kTmaEntryBytes == 16) sts128u(a, e);
      else asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(e.x), "r"(e.z) : "memory");
    };
    static_for<0, RW>([&](auto ic) {
      constexpr int i = decltype(ic)::value;
      acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
      const int64_t r = r0 + wp * RW + i;
      const bool valid = r < A.rows;
      const int rbeg = valid ? __ldg(A.ptr + r) : 0;
      const int rend = valid ? __ldg(A.ptr + r + 1) : 0;
      if (lane == 0) s_span[wp][i] = make_int2(rbeg, rend);
      k[i] = 0;
      uint4 ent;
      load_entry(rbeg, rend, cl[i], ent);
      ent_store(ent0 + (i * 32 + lane) * kTmaEntryBytes, ent);
      prefetch_next(rbeg, rend);
    });
    __syncwarp();

    const uint32_t lane_off = (uint32_t)(lane * 4 * E);
    for (int64_t ch = 0; ch < nchunks; ++ch) {
      const int st = (int)(ch % kTmaStages);
      bool ok = s_abort == 0 && mbar_wait_bounded(full0 + 8 * st, (uint32_t)((ch / kTmaStages) & 1), limit_ns);
      ok = __all_sync(kFull, ok);
      if (!ok) {
        if (lane == 0) s_abort = 1;
        break;
      }
      const int64_t kc = ch * KC;
      // dense row c of this chunk (this lane's 4 columns) sits at xoff + c * ROWB
      const uint32_t xoff = xs + (uint32_t)(st * CHUNK) + lane_off - (uint32_t)(kc * ROWB);
      const int cbound = (int)mn64(kc + KC, A.brows);  // columns below it are staged
      static_for<0, RW>([&](auto ic) {
        constexpr int i = decltype(ic)::value;
        const uint32_t eb = ent0 + i * 32 * kTmaEntryBytes;
        auto ent_load = [&](int tt) -> uint4 {
          if constexpr (kTmaEntryBytes == 16) {
            return lds128u(eb + tt * 16);
          } else {
            const uint2 w = lds64(eb + tt * 8);
            return make_uint4(w.x, w.x, w.y, 0u);
          }
        };
        float2 a01 = acc[i][0], a23 = acc[i][1];
        auto fma_x = [&](const uint4& e, const float4& x) {
          const float2 vv = make_float2(__uint_as_float(e.x), __uint_as_float(e.y));
          a01 = __ffma2_rn(vv, make_float2(x.x, x.y), a01);
          a23 = __ffma2_rn(vv, make_float2(x.z, x.w), a23);
        };
        auto load_x = [&](const uint4& e) -> float4 {
          if constexpr (E == 4) {
            return lds128(xoff + e.z);
          } else {
            const uint2 w = lds64(xoff + e.z);
            return make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
          }
        };
        while (true) {
          const int lim = __popc(__ballot_sync(kFull, cl[i] < cbound));  // sorted: a prefix
          int t = k[i];
          for (; t + 4 <= lim; t += 4) {
            uint4 e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) e[u] = ent_load(t + u);
            float4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = load_x(e[u]);
            if constexpr (E == 2 || RW <= 6) {
              // two FMA chains of two (odd entries into b01/b23), joined by one packed add
              float2 b01 = make_float2(0.f, 0.f), b23 = make_float2(0.f, 0.f);
#pragma unroll
              for (int u = 0; u < 4; u += 2) {
                const float2 v0 = make_float2(__uint_as_float(e[u].x), __uint_as_float(e[u].y));
                const float2 v1 = make_float2(__uint_as_float(e[u + 1].x), __uint_as_float(e[u + 1].y));
                a01 = __ffma2_rn(v0, make_float2(x[u].x, x[u].y), a01);
                a23 = __ffma2_rn(v0, make_float2(x[u].z, x[u].w), a23);
                b01 = __ffma2_rn(v1, make_float2(x[u + 1].x, x[u + 1].y), b01);
                b23 = __ffma2_rn(v1, make_float2(x[u + 1].z, x[u + 1].w), b23);
              }
              a01 = __fadd2_rn(a01, b01);
              a23 = __fadd2_rn(a23, b23);
            } else {  // fp32 with 8 rows per warp: no registers to spare for a second chain
#pragma unroll
              for (int u = 0; u < 4; ++u) fma_x(e[u], x[u]);
            }
          }
          if (t < lim) {  // up to three more: predicated loads first, then the FMAs
            uint4 e[3];
            float4 x[3];
#pragma unroll
            for (int u = 0; u < 3; ++u) {
              e[u] = make_uint4(0u, 0u, 0u, 0u);
              x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 3; ++u)
              if (t + u < lim) e[u] = ent_load(t + u);
#pragma unroll
            for (int u = 0; u < 3; ++u)
              if (t + u < lim) x[u] = load_x(e[u]);
#pragma unroll
            for (int u = 0; u < 3; ++u)
              if (t + u < lim) fma_x(e[u], x[u]);
          }
          k[i] = lim;
          if (lim < 32) break;  // the rest of the batch lies beyond this chunk (or the row)
          // the batch is used up: load the next one (prefetched into L1) and the one after
          const int2 sp = s_span[wp][i];
          const int nb = sp.x + 32;
          uint4 ent;
          load_entry(nb, sp.y, cl[i], ent);
          __syncwarp();
          ent_store(eb + lane * kTmaEntryBytes, ent);
          if (lane == 0) s_span[wp][i].x = nb;
          __syncwarp();
          k[i] = 0;
          prefetch_next(nb, sp.y);
        }
        acc[i][0] = a01;
        acc[i][1] = a23;
      });
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);  // this warp is done with the stage
    }
  }
  __syncthreads();  // every role has finished (all waits above are bounded)
  if (s_abort) {    // a wait gave up: report, let the issued copies land (bounded), return
    if (wp == kTmaConsumers && lane == 0) {
      if (A.err) atomicOr(A.err, ERRBIT_TIMEOUT);
      // the last phase issued into each stage (earlier ones completed before it was reissued)
      for (int64_t ch = mn64(issued, nchunks) - 1; ch >= 0 && ch >= issued - kTmaStages; --ch)
        mbar_wait_bounded(full0 + 8 * (int)(ch % kTmaStages), (uint32_t)((ch / kTmaStages) & 1), limit_ns);
    }
    return;
  }
  if (wp == kTmaConsumers) return;

  const int c0 = lane * 4;
  static_for<0, RW>([&](auto ic) {
    constexpr int i = decltype(ic)::value;
    const int64_t r = r0 + wp * RW + i;
    if (r < A.rows && c0 < ncols) {
      const float a[4] = {acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y};
      T* dst = A.C + r * A.ldc + n0 + c0;
      if (c0 + 4 <= ncols && ((uintptr_t)dst % (4 * E)) == 0) {  // one vector store where aligned
        store_cols<4>(dst, a);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < ncols - c0) store1(dst + j, a[j]);
      }
    }
  });
}

// ------------------------------------------------------------------------- zero fill

template <typename T>
__global__ void k_zero_rows(T* C, int64_t rows, int64_t N, int64_t ldc) {
  const int64_t total = rows * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    store1(C + (i / N) * ldc + (i % N), 0.f);
}

// ------------------------------------------------------------------------- host dispatch

int pow2ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

bool aligned(const void* p, int64_t ld, int nc, int elem) {
  return ((uintptr_t)p % (uintptr_t)(nc * elem)) == 0 && (ld % nc) == 0;
}

// Widest per-lane group (<= 32 bytes, in vectors of <= 16 bytes) that divides `ncols`
// and keeps every listed row aligned for its vector loads.
int pick_nc(int ncols, int elem, const void* p0, int64_t ld0, const void* p1, int64_t ld1) {
  int nc = 32 / elem;
  auto ok = [&](int c) {
    const int vec = std::min(c, 16 / elem);  // elements per vector access
    return (ncols % c) == 0 && aligned(p0, ld0, vec, elem) && aligned(p1, ld1, vec, elem);
  };
  while (nc > 1 && !ok(nc)) nc >>= 1;
  return nc;
}

// cudaFuncSetAttribute for a kernel's dynamic shared memory above 48 KB, once per device.
template <auto Kern>
cudaError_t ensure_dynamic_smem(int bytes) {
  constexpr int kDev = 64;
  static std::once_flag once[kDev];
  static cudaError_t result[kDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kDev) return cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  std::call_once(once[dev], [&] {
    result[dev] = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return result[dev];
}

// The driver's tensor-map encoder, looked up once through the runtime (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map of the dense operand B (brows x N, leading dimension ldb) for boxes of
// box_rows rows x kWideCols columns; false where TMA's rules (16-byte aligned base and row
// stride) or the driver rule it out.
template <typename T>
bool dense_tensor_map(CUtensorMap* map, const T* B, int64_t brows, int64_t N, int64_t ldb, int box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr || ((uintptr_t)B % 16) != 0 || ((ldb * (int64_t)sizeof(T)) % 16) != 0) return false;
  if (brows <= 0 || N <= 0 || brows >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31)) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)brows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ldb * (int64_t)sizeof(T))};
  const cuuint32_t box[2] = {(cuuint32_t)kWideCols, (cuuint32_t)box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUtensorMapDataType dt =
      sizeof(T) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(map, dt, 2, const_cast<T*>(B), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Args>
cudaError_t launch_pdl(void (*kern)(const Args), dim3 grid, cudaStream_t s, const Args& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args);
}

template <typename T, bool TRANS, typename I>
using SpmmKernel = void (*)(const SpmmArgs<T, I>);

// Instantiated shapes: 32-byte groups (NC = 16 bf16 / 8 fp32) with G = 1..64/NC lanes,
// 16-byte groups with one or two lanes (two when a 32-byte operand row is split between
// them), 8- and 4-byte groups with one lane, and scalars with G = 1..32.
template <typename T, bool TRANS, typename I>
SpmmKernel<T, TRANS, I> pick_spmm(int nc, int g) {
#define SNK_CASE(NC_, G_) \
  if (nc == NC_ && g == G_) return k_spmm_small<T, NC_, G_, TRANS, I>;
  if constexpr (sizeof(T) == 2) {
    SNK_CASE(16, 1) SNK_CASE(16, 2) SNK_CASE(16, 4)
    SNK_CASE(8, 1) SNK_CASE(8, 2) SNK_CASE(4, 1) SNK_CASE(2, 1)
  } else {
    SNK_CASE(8, 1) SNK_CASE(8, 2) SNK_CASE(8, 4) SNK_CASE(8, 8)
    SNK_CASE(4, 1) SNK_CASE(4, 2) SNK_CASE(2, 1)
  }
  SNK_CASE(1, 1) SNK_CASE(1, 2) SNK_CASE(1, 4) SNK_CASE(1, 8) SNK_CASE(1, 16) SNK_CASE(1, 32)
#undef SNK_CASE
  return nullptr;
}

template <typename T, typename I>
using SddmmKernel = void (*)(const SddmmArgs<T, I>);

template <typename T, typename I>
SddmmKernel<T, I> pick_sddmm(int nc, int g, bool deep) {
  if (deep && g == 32 && nc * (int)sizeof(T) == 32) return k_sddmm_small<T, 32 / (int)sizeof(T), 32, I, true>;
#define SNK_CASE(NC_, G_) \
  if (nc == NC_ && g == G_) return k_sddmm_small<T, NC_, G_, I, false>;
  if constexpr (sizeof(T) == 2) {
    SNK_CASE(16, 1) SNK_CASE(16, 2) SNK_CASE(16, 4) SNK_CASE(16, 8) SNK_CASE(16, 16) SNK_CASE(16, 32)
    SNK_CASE(8, 1) SNK_CASE(4, 1) SNK_CASE(2, 1)
  } else {
    SNK_CASE(8, 1) SNK_CASE(8, 2) SNK_CASE(8, 4) SNK_CASE(8, 8) SNK_CASE(8, 16) SNK_CASE(8, 32)
    SNK_CASE(4, 1) SNK_CASE(2, 1)
  }
  SNK_CASE(1, 1) SNK_CASE(1, 2) SNK_CASE(1, 4) SNK_CASE(1, 8) SNK_CASE(1, 16) SNK_CASE(1, 32)
#undef SNK_CASE
  return nullptr;
}

// Test hook for the bounded waits: SNK_TEST_TMA_EXTRA_TX=<bytes> in the environment makes
// every chunk expect that many bytes more than its copy delivers, so no "full" barrier ever
// completes and every wait of the kernel runs out (about a second each); the kernel then
// reports ERRBIT_TIMEOUT and returns.  Nothing faults and no copy is left in flight.  Unset
// (the normal case) it is 0.
uint32_t tma_test_extra_tx() {
  const char* e = std::getenv("SNK_TEST_TMA_EXTRA_TX");
  if (e == nullptr) return 0u;
  const long v = std::strtol(e, nullptr, 10);
  return (v > 0 && v <= 4096) ? (uint32_t)v : 0u;
}

// The TMA-staged wide kernel; SNK_ERR_UNSUPPORTED (nothing launched) where no tensor map
// can describe B, so that the caller takes another path.
template <typename T, bool TRANS, int RW, typename I>
snk_status launch_tma(const WideArgs<T, I>& A, const T* B, int64_t N, int64_t ldb, int64_t slices, cudaStream_t s) {
  constexpr int kc = tma_kc<T, RW>();
  CUtensorMap map;
  if (!dense_tensor_map<T>(&map, B, A.brows, N, ldb, kc)) return SNK_ERR_UNSUPPORTED;
  const int smem = kTmaStages * kc * kWideCols * (int)sizeof(T) + 128;  // + room to align the ring
  const int rb = kTmaConsumers * RW;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((A.rows + rb - 1) / rb), (unsigned)slices);
  cfg.blockDim = dim3(kTmaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SNK_CUDA_TRY((ensure_dynamic_smem<k_spmm_tma<T, TRANS, RW, I>>(smem)));
  SNK_CUDA_TRY((cudaLaunchKernelEx(&cfg, k_spmm_tma<T, TRANS, RW, I>, A, map)));
  return SNK_OK;
}

template <typename T, bool TRANS, typename I>
snk_status spmm_tma(const snk_layout* L, const I* idx, const T* values, const T* B, int64_t N, int64_t ldb, T* C,
                    int64_t ldc, cudaStream_t s) {
  WideArgs<T, I> A;
  A.ptr = TRANS ? L->col_ptr : L->row_ptr;
  A.idx = idx;
  A.perm = TRANS ? L->perm : nullptr;
  A.vals = values;
  A.B = B;
  A.C = C;
  A.ldb = ldb;
  A.ldc = ldc;
  A.rows = TRANS ? L->K : L->M;
  A.brows = TRANS ? L->M : L->K;
  A.N = (int)N;
  A.err = L->err;
  A.extra_tx = tma_test_extra_tx();
  const int64_t slices = (N + kWideCols - 1) / kWideCols;
  if (N >= ((int64_t)1 << 31) || slices > 65535) return SNK_ERR_UNSUPPORTED;
  // rows per consumer warp: the choice among 8, 6 and 4 with the shortest estimated
  // makespan, rounds of two CTAs per SM x (rows per warp + a staging term)
  const int64_t slots = 2 * (int64_t)std::max(L->sm_count, 1);
  int best = 8;
  int64_t best_cost = -1;
  for (int rw : {8, 6, 4}) {
    const int64_t tiles = ((A.rows + 8 * rw - 1) / (8 * rw)) * slices;
    const int64_t cost = ((tiles + slots - 1) / slots) * (rw + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = rw;
    }
  }
  if (best == 8) return launch_tma<T, TRANS, 8, I>(A, B, N, ldb, slices, s);
  if (best == 6) return launch_tma<T, TRANS, 6, I>(A, B, N, ldb, slices, s);
  return launch_tma<T, TRANS, 4, I>(A, B, N, ldb, slices, s);
}

template <typename T, bool TRANS, typename I>
snk_status spmm_typed(const snk_layout* L, const I* idx, const T* values, const T* B, int64_t N, int64_t ldb, T* C,
                      int64_t ldc, cudaStream_t s) {
  const int elem = (int)sizeof(T);
  const int64_t rows = TRANS ? L->K : L->M;
  // wide operands: the TMA-staged row-block x column-slice kernel where a tensor map can
  // describe B (16-byte aligned base and row stride)
  if (N >= kTmaMinN) {
    const snk_status st = spmm_tma<T, TRANS, I>(L, idx, values, B, N, ldb, C, ldc, s);
    if (st != SNK_ERR_UNSUPPORTED) return st;
  }
  for (int64_t col0 = 0; col0 < N; col0 += kCarryCols) {
    const int ncols = (int)std::min<int64_t>(kCarryCols, N - col0);
    const T* Bc = B + col0;
    T* Cc = C + col0;
    int nc = pick_nc(ncols, elem, Bc, ldb, Cc, ldc);
    int g = pow2ceil((ncols + nc - 1) / nc);
    const int gmax = nc == 1 ? 32 : (nc * elem == 32 ? 64 / nc : 1);
    if (g > gmax) {  // narrow vectors come with one lane only: use scalars instead
      nc = 1;
      g = pow2ceil(ncols);
    }
    g = std::min(g, 32);
    if (g == 1 && nc * elem == 32) {  // a one-lane worker of 32 bytes: two lanes of 16 (measured faster)
      nc /= 2;
      g = 2;
    }
    const int nt = nc * g;
    const int tiles = (ncols + nt - 1) / nt;
    auto kern = pick_spmm<T, TRANS, I>(nc, g);
    if (kern == nullptr || tiles > kMaxTiles) return SNK_ERR_UNSUPPORTED;
    SpmmArgs<T, I> A;
    A.ptr = TRANS ? L->col_ptr : L->row_ptr;
    A.idx = idx;
    A.perm = TRANS ? L->perm : nullptr;
    A.vals = values;
    A.desc = TRANS ? L->desc_t : L->desc_f;
    A.B = Bc;
    A.C = Cc;
    A.ldb = ldb;
    A.ldc = ldc;
    A.rows = rows;
    A.nnz = L->nnz;
    A.P = L->P;
    A.ncols = ncols;
    A.b32 = (TRANS ? L->M : L->K) * ldb <= (int64_t)0xffffffffLL ? 1 : 0;
    A.a32 = (nc * elem == 32 && ((uintptr_t)Bc % 32) == 0 && ((ldb * elem) % 32) == 0) ? 1 : 0;
    A.bbytes = (ldb == ncols) ? (TRANS ? L->M : L->K) * ldb * elem : 0;
    A.prows = rows + 1;
    A.carry_tail = TRANS ? L->carry_tail_b : L->carry_tail_f;
    A.carry_head = TRANS ? L->carry_head_b : L->carry_head_f;
    A.cnt = TRANS ? L->cnt_b : L->cnt_f;
    SNK_CUDA_TRY(launch_pdl(kern, dim3((unsigned)L->P, (unsigned)tiles), s, A));
  }
  return SNK_OK;
}

template <typename T, typename I>
snk_status sddmm_typed(const snk_layout* L, const I* col, const T* dY, int64_t lddy, const T* X, int64_t ldx,
                       int64_t N, T* dW, cudaStream_t s) {
  const int elem = (int)sizeof(T);
  const int ncap = (int)std::min<int64_t>(N, 1 << 20);
  int nc = pick_nc(std::max(ncap, 1), elem, X, ldx, dY, lddy);
  int g = (int)std::min<int64_t>(32, pow2ceil((int)std::min<int64_t>((N + nc - 1) / nc, 64)));
  auto kern = pick_sddmm<T, I>(nc, g, N >= 256);
  if (kern == nullptr) {
    nc = 1;
    g = (int)std::min<int64_t>(32, pow2ceil((int)std::max<int64_t>(1, std::min<int64_t>(N, 64))));
    kern = pick_sddmm<T, I>(nc, g, false);
  }
  if (kern == nullptr) return SNK_ERR_UNSUPPORTED;
  SddmmArgs<T, I> A;
  A.row_ptr = L->row_ptr;
  A.col = col;
  A.desc = L->desc_f;
  A.X = X;
  A.dY = dY;
  A.dW = dW;
  A.ldx = ldx;
  A.lddy = lddy;
  A.rows = L->M;
  A.nnz = L->nnz;
  A.N = (int)N;
  A.a32 = (nc * elem == 32 && ((uintptr_t)X % 32) == 0 && ((uintptr_t)dY % 32) == 0 && ((ldx * elem) % 32) == 0 &&
           ((lddy * elem) % 32) == 0) ? 1 : 0;
  A.xbytes = ldx == N ? L->K * N * elem : 0;
  A.dybytes = lddy == N ? L->M * N * elem : 0;
  SNK_CUDA_TRY(launch_pdl(kern, dim3((unsigned)L->P), s, A));
  return SNK_OK;
}

}  // namespace

snk_status launch_zero_rows(void* C, int64_t rows, int64_t N, int64_t ldc, int elem_bytes, cudaStream_t s) {
  if (rows <= 0 || N <= 0) return SNK_OK;
  const int64_t total = rows * N;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, 65535 * 4);
  if (elem_bytes == 4)
    k_zero_rows<float><<<grid, 256, 0, s>>>((float*)C, rows, N, ldc);
  else
    k_zero_rows<__nv_bfloat16><<<grid, 256, 0, s>>>((__nv_bfloat16*)C, rows, N, ldc);
  SNK_CUDA_TRY(cudaGetLastError());
  return SNK_OK;
}

namespace {

// Entry points by value type and index width: the 16-bit copies of the index arrays are
// used when the layout is switched to them (and holds them).
template <typename T>
snk_status spmm_by_index(const snk_layout* L, bool transpose, const T* values, const T* B, int64_t N, int64_t ldb,
                         T* C, int64_t ldc, cudaStream_t s) {
  if (L->index_bits == 16 && L->col16 != nullptr && L->csc_row16 != nullptr) {
    return transpose ? spmm_typed<T, true, uint16_t>(L, L->csc_row16, values, B, N, ldb, C, ldc, s)
                     : spmm_typed<T, false, uint16_t>(L, L->col16, values, B, N, ldb, C, ldc, s);
  }
  return transpose ? spmm_typed<T, true, int32_t>(L, L->csc_row, values, B, N, ldb, C, ldc, s)
                   : spmm_typed<T, false, int32_t>(L, L->col, values, B, N, ldb, C, ldc, s);
}

template <typename T>
snk_status sddmm_by_index(const snk_layout* L, const T* dY, int64_t lddy, const T* X, int64_t ldx, int64_t N, T* dW,
                          cudaStream_t s) {
  if (L->index_bits == 16 && L->col16 != nullptr)
    return sddmm_typed<T, uint16_t>(L, L->col16, dY, lddy, X, ldx, N, dW, s);
  return sddmm_typed<T, int32_t>(L, L->col, dY, lddy, X, ldx, N, dW, s);
}

}  // namespace

snk_status launch_spmm(const snk_layout* L, bool transpose, const void* values, const void* B, int64_t N, int64_t ldb,
                       void* C, int64_t ldc, cudaStream_t s) {
  const int64_t rows = transpose ? L->K : L->M;
  if (L->nnz == 0) return launch_zero_rows(C, rows, N, ldc, L->dtype == SNK_F32 ? 4 : 2, s);
  if (L->dtype == SNK_F32)
    return spmm_by_index<float>(L, transpose, (const float*)values, (const float*)B, N, ldb, (float*)C, ldc, s);
  using bf = __nv_bfloat16;
  return spmm_by_index<bf>(L, transpose, (const bf*)values, (const bf*)B, N, ldb, (bf*)C, ldc, s);
}

snk_status launch_sddmm(const snk_layout* L, const void* dY, int64_t lddy, const void* X, int64_t ldx, int64_t N,
                        void* dW, cudaStream_t s) {
  if (L->nnz == 0) return SNK_OK;
  if (L->dtype == SNK_F32)
    return sddmm_by_index<float>(L, (const float*)dY, lddy, (const float*)X, ldx, N, (float*)dW, s);
  using bf = __nv_bfloat16;
  return sddmm_by_index<bf>(L, (const bf*)dY, lddy, (const bf*)X, ldx, N, (bf*)dW, s);
}

}  // namespace snk
