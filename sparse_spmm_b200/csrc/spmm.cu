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
// A lane holds up to 32 bytes of a row (two 16-byte vector loads), so few lanes repeat
// the per-entry index and value loads.
#include <algorithm>

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
__device__ __forceinline__ void load_packed(const T* p, Packed<T, NC>& r) {
  constexpr int W = Packed<T, NC>::W;
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

// acc[j] += v * x[j] for the NC columns, two columns per packed fp32 FMA.
template <typename T, int NC>
__device__ __forceinline__ void fma_row(float v, const Packed<T, NC>& x, float* acc) {
  if constexpr (NC == 1) {
    acc[0] = fmaf(v, unpack<T, NC>(x, 0), acc[0]);
  } else {
    const float2 vv = make_float2(v, v);
#pragma unroll
    for (int j = 0; j < NC; j += 2) {
      float2 a2 = make_float2(acc[j], acc[j + 1]);
      a2 = __ffma2_rn(vv, make_float2(unpack<T, NC>(x, j), unpack<T, NC>(x, j + 1)), a2);
      acc[j] = a2.x;
      acc[j + 1] = a2.y;
    }
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

template <typename T>
struct SpmmArgs {
  const int32_t* ptr;  // [rows + 1] row_ptr (forward) or col_ptr (transposed)
  const int32_t* idx;  // [nnz] col (forward) or csc_row (transposed)
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
  float* carry_tail;   // [P][kCarryCols]
  float* carry_head;   // [P][kCarryCols]
  uint32_t* cnt;       // [kMaxTiles][P], zero between launches
};

// Entries in flight per worker: as many as the register budget of 3 CTAs per SM allows.
template <typename T, int NC>
constexpr int spmm_batch() { return NC * (int)sizeof(T) >= 32 ? 3 : (NC * (int)sizeof(T) >= 16 ? 6 : 8); }
template <typename T, int NC>
constexpr int sddmm_batch() { return NC * (int)sizeof(T) >= 32 ? 2 : (NC * (int)sizeof(T) >= 8 ? 4 : 6); }

template <typename T, int NC, int G, bool TRANS>
__global__ void __launch_bounds__(kThreads, 3) k_spmm_small(const SpmmArgs<T> A) {
  constexpr int NW = kThreads / G;   // workers per CTA
  constexpr int WPW = 32 / G;        // workers per warp
  constexpr int NT = NC * G;         // columns per tile
  constexpr int NWARPS = kThreads / 32;
  constexpr int UB = spmm_batch<T, NC>();
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
  pdl_wait();

  const int4 dsc = __ldg(A.desc + part);
  const int64_t a = dsc.x, b = dsc.y, ra = dsc.z, rb = dsc.w;
  const int np = (int)(b - a);
  // the worker's piece, as offsets from a
  const int s = (int)(((int64_t)np * w) / NW);
  const int e_end = (int)(((int64_t)np * (w + 1)) / NW);
  const int32_t* __restrict__ idx = A.idx + a;
  const int32_t* __restrict__ prm = TRANS ? A.perm + a : nullptr;
  const T* __restrict__ vals = TRANS ? A.vals : A.vals + a;

  // the worker's next batch of indices / values (prefetched one batch ahead)
  int c[UB];
  float v[UB];
  auto load_batch = [&](int e0, int nb) {
#pragma unroll
    for (int i = 0; i < UB; ++i) {
      if (i < nb) {
        c[i] = __ldg(idx + e0 + i);
        v[i] = TRANS ? load1(vals + __ldg(prm + e0 + i)) : load1(vals + e0 + i);
      }
    }
  };
  if (s < e_end) load_batch(s, min(UB, e_end - s));

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

  float acc[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) acc[j] = 0.f;
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
#pragma unroll
      for (int j = 0; j < NC; ++j) acc[j] = 0.f;
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
          load_packed<NC>(src, x[i]);
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
  float H[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) H[j] = 0.f;  // holds the incoming prefix until it is added
  for (int q = 0; q < wp; ++q) {
    const int fq = s_aggF[q];
#pragma unroll
    for (int j = 0; j < NC; ++j) H[j] = fq ? s_agg[q][l * NC + j] : H[j] + s_agg[q][l * NC + j];
  }
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
    if (RP(t + 1) > np) cross_cta(t, acc, false);
  }
}

// ------------------------------------------------------------------------- SDDMM

template <typename T>
struct SddmmArgs {
  const int32_t* row_ptr;
  const int32_t* col;
  const int4* desc;  // [P] per-CTA work descriptors (forward ones)
  const T* X;        // K x N
  const T* dY;       // M x N
  T* dW;             // [nnz]
  int64_t ldx, lddy;
  int64_t rows;
  int64_t nnz;
  int N;             // a multiple of NC
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

template <typename T, int NC, int G>
__global__ void __launch_bounds__(kThreads, 3) k_sddmm_small(const SddmmArgs<T> A) {
  constexpr int NW = kThreads / G;
  constexpr int NT = NC * G;
  constexpr int UB = sddmm_batch<T, NC>();
  __shared__ int32_t s_rp[kRowCap];
  __shared__ float s_dw[kStageCap];

  pdl_launch_dependents();
  const int part = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int w = tid / G, l = tid % G;
  const int lane_base = lane - l;
  const unsigned gmask = G == 32 ? kFull : (((1u << G) - 1u) << lane_base);
  pdl_wait();

  const int4 dsc = __ldg(A.desc + part);
  const int64_t a = dsc.x, b = dsc.y, ra = dsc.z, rb = dsc.w;
  const int np = (int)(b - a);
  const bool staged = np <= kStageCap;
  const int s = (int)(((int64_t)np * w) / NW);
  const int e_end = (int)(((int64_t)np * (w + 1)) / NW);
  const int32_t* __restrict__ col = A.col + a;
  int c[UB];
  auto load_batch = [&](int e0, int nb) {
#pragma unroll
    for (int i = 0; i < UB; ++i)
      if (i < nb) c[i] = __ldg(col + e0 + i);
  };
  if (s < e_end) load_batch(s, min(UB, e_end - s));
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
          if (i < nb) load_packed<NC>(A.X + (int64_t)cc[i] * A.ldx + n0, xv[i]);
        if (one_row) {
          Packed<T, NC> yv;
          load_packed<NC>(A.dY + (int64_t)rr[0] * A.lddy + n0, yv);
#pragma unroll
          for (int i = 0; i < UB; ++i)
            if (i < nb) d[i] = dot_packed(xv[i], yv, d[i]);
        } else {
#pragma unroll
          for (int i = 0; i < UB; ++i) {
            if (i < nb) {
              Packed<T, NC> yv;
              load_packed<NC>(A.dY + (int64_t)rr[i] * A.lddy + n0, yv);
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

template <typename T, bool TRANS>
using SpmmKernel = void (*)(const SpmmArgs<T>);

// Instantiated shapes: 32-byte groups (NC = 16 bf16 / 8 fp32) with G = 1..64/NC lanes,
// 16-, 8- and 4-byte groups with one lane, and scalars with G = 1..32.
template <typename T, bool TRANS>
SpmmKernel<T, TRANS> pick_spmm(int nc, int g) {
#define SNK_CASE(NC_, G_) \
  if (nc == NC_ && g == G_) return k_spmm_small<T, NC_, G_, TRANS>;
  if constexpr (sizeof(T) == 2) {
    SNK_CASE(16, 1) SNK_CASE(16, 2) SNK_CASE(16, 4)
    SNK_CASE(8, 1) SNK_CASE(4, 1) SNK_CASE(2, 1)
  } else {
    SNK_CASE(8, 1) SNK_CASE(8, 2) SNK_CASE(8, 4) SNK_CASE(8, 8)
    SNK_CASE(4, 1) SNK_CASE(2, 1)
  }
  SNK_CASE(1, 1) SNK_CASE(1, 2) SNK_CASE(1, 4) SNK_CASE(1, 8) SNK_CASE(1, 16) SNK_CASE(1, 32)
#undef SNK_CASE
  return nullptr;
}

template <typename T>
using SddmmKernel = void (*)(const SddmmArgs<T>);

template <typename T>
SddmmKernel<T> pick_sddmm(int nc, int g) {
#define SNK_CASE(NC_, G_) \
  if (nc == NC_ && g == G_) return k_sddmm_small<T, NC_, G_>;
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

template <typename T, bool TRANS>
snk_status spmm_typed(const snk_layout* L, const T* values, const T* B, int64_t N, int64_t ldb, T* C, int64_t ldc,
                      cudaStream_t s) {
  const int elem = (int)sizeof(T);
  const int64_t rows = TRANS ? L->K : L->M;
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
    const int nt = nc * g;
    const int tiles = (ncols + nt - 1) / nt;
    auto kern = pick_spmm<T, TRANS>(nc, g);
    if (kern == nullptr || tiles > kMaxTiles) return SNK_ERR_UNSUPPORTED;
    SpmmArgs<T> A;
    A.ptr = TRANS ? L->col_ptr : L->row_ptr;
    A.idx = TRANS ? L->csc_row : L->col;
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
    A.carry_tail = TRANS ? L->carry_tail_b : L->carry_tail_f;
    A.carry_head = TRANS ? L->carry_head_b : L->carry_head_f;
    A.cnt = TRANS ? L->cnt_b : L->cnt_f;
    SNK_CUDA_TRY(launch_pdl(kern, dim3((unsigned)L->P, (unsigned)tiles), s, A));
  }
  return SNK_OK;
}

template <typename T>
snk_status sddmm_typed(const snk_layout* L, const T* dY, int64_t lddy, const T* X, int64_t ldx, int64_t N, T* dW,
                       cudaStream_t s) {
  const int elem = (int)sizeof(T);
  const int ncap = (int)std::min<int64_t>(N, 1 << 20);
  int nc = pick_nc(std::max(ncap, 1), elem, X, ldx, dY, lddy);
  int g = (int)std::min<int64_t>(32, pow2ceil((int)std::min<int64_t>((N + nc - 1) / nc, 64)));
  auto kern = pick_sddmm<T>(nc, g);
  if (kern == nullptr) {
    nc = 1;
    g = (int)std::min<int64_t>(32, pow2ceil((int)std::max<int64_t>(1, std::min<int64_t>(N, 64))));
    kern = pick_sddmm<T>(nc, g);
  }
  if (kern == nullptr) return SNK_ERR_UNSUPPORTED;
  SddmmArgs<T> A;
  A.row_ptr = L->row_ptr;
  A.col = L->col;
  A.desc = L->desc_f;
  A.X = X;
  A.dY = dY;
  A.dW = dW;
  A.ldx = ldx;
  A.lddy = lddy;
  A.rows = L->M;
  A.nnz = L->nnz;
  A.N = (int)N;
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

snk_status launch_spmm(const snk_layout* L, bool transpose, const void* values, const void* B, int64_t N, int64_t ldb,
                       void* C, int64_t ldc, cudaStream_t s) {
  const int64_t rows = transpose ? L->K : L->M;
  if (L->nnz == 0) return launch_zero_rows(C, rows, N, ldc, L->dtype == SNK_F32 ? 4 : 2, s);
  if (L->dtype == SNK_F32) {
    return transpose ? spmm_typed<float, true>(L, (const float*)values, (const float*)B, N, ldb, (float*)C, ldc, s)
                     : spmm_typed<float, false>(L, (const float*)values, (const float*)B, N, ldb, (float*)C, ldc, s);
  }
  using bf = __nv_bfloat16;
  return transpose ? spmm_typed<bf, true>(L, (const bf*)values, (const bf*)B, N, ldb, (bf*)C, ldc, s)
                   : spmm_typed<bf, false>(L, (const bf*)values, (const bf*)B, N, ldb, (bf*)C, ldc, s);
}

snk_status launch_sddmm(const snk_layout* L, const void* dY, int64_t lddy, const void* X, int64_t ldx, int64_t N,
                        void* dW, cudaStream_t s) {
  if (L->nnz == 0) return SNK_OK;
  if (L->dtype == SNK_F32)
    return sddmm_typed<float>(L, (const float*)dY, lddy, (const float*)X, ldx, N, (float*)dW, s);
  using bf = __nv_bfloat16;
  return sddmm_typed<bf>(L, (const bf*)dY, lddy, (const bf*)X, ldx, N, (bf*)dW, s);
}

}  // namespace snk
