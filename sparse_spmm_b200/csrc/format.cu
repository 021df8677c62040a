// format.cu -- COO format work on the GPU: validation, the (row, col) sort, row pointers,
// the CSC permutation, nnz-balanced partitions, and connection restructuring.
//
// The pages ("Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural Networks on GPU",
// arXiv 2610.04093, Abstract) fix only that the layer is held as COO and that connections
// can be restructured.  Everything here is integer work and must be bit-exact: the sorted
// order is unique because duplicate positions are rejected, so any correct sort agrees.
//
// Sorting is a stable least-significant-digit radix sort over 8-bit digits (3 kernels per
// pass: per-tile digit histograms, one exclusive scan, a stable scatter that ranks equal
// digits inside a warp with __match_any_sync).
#include <algorithm>

#include "internal.cuh"

namespace snk {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanTile = kScanThreads * kScanItems;

int grid_for(int64_t n, int threads, int cap = 65535 * 4) {
  int64_t g = ceil_div(std::max<int64_t>(n, 1), threads);
  return (int)std::min<int64_t>(g, cap);
}

int bits_for(uint64_t maxval) {
  int b = 0;
  while (b < 64 && (maxval >> b) != 0) ++b;
  return b;
}

// ------------------------------------------------------------------------- basic kernels

__global__ void k_fill_u32(uint32_t* p, int64_t n, uint32_t v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

template <typename W>
__global__ void k_copy(const W* __restrict__ src, W* __restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

__global__ void k_iota_i32(int32_t* p, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = (int32_t)i;
}

// ------------------------------------------------------------------------- radix sort

__global__ void __launch_bounds__(kSortThreads) k_rs_hist(const uint64_t* __restrict__ keys, int64_t n, int shift,
                                                          uint32_t* __restrict__ hist, int nblocks) {
  __shared__ uint32_t h[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kSortTile;
  for (int i = threadIdx.x; i < kSortTile; i += blockDim.x) {
    int64_t j = base + i;
    if (j < n) atomicAdd(&h[(uint32_t)(keys[j] >> shift) & 255u], 1u);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[(int64_t)d * nblocks + blockIdx.x] = h[d];
}

// Stable scatter of one 8-bit digit.  Warp w of a block owns the 256 consecutive keys
// [tile + 256 w, tile + 256 (w + 1)), visited 32 at a time in order, so the order of equal
// digits is: by warp, then by round, then by lane -- i.e. the input order.
__global__ void __launch_bounds__(kSortThreads) k_rs_scatter(const uint64_t* __restrict__ kin,
                                                             const uint32_t* __restrict__ vin,
                                                             uint64_t* __restrict__ kout,
                                                             uint32_t* __restrict__ vout, int64_t n, int shift,
                                                             const uint32_t* __restrict__ offs, int nblocks) {
  constexpr int kWarps = kSortThreads / 32;
  __shared__ uint32_t wc[kWarps][256];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int i = tid; i < kWarps * 256; i += kSortThreads) (&wc[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kSortTile + (int64_t)w * (kSortItems * 32);
  const uint32_t lt = (1u << lane) - 1u;
  uint64_t k[kSortItems];
  uint32_t v[kSortItems], d[kSortItems], lr[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t j = base + r * 32 + lane;
    const bool valid = j < n;
    uint32_t dig = 256u + (uint32_t)lane;  // unique dummy digit for lanes past the end
    k[r] = 0;
    v[r] = 0;
    if (valid) {
      k[r] = kin[j];
      v[r] = vin[j];
      dig = (uint32_t)(k[r] >> shift) & 255u;
    }
    d[r] = dig;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig);
    const uint32_t rank = __popc(peers & lt);
    uint32_t cnt = 0;
    if (valid) cnt = wc[w][dig];
    __syncwarp();
    if (valid && rank == 0) wc[w][dig] = cnt + __popc(peers);
    __syncwarp();
    lr[r] = cnt + rank;
  }
  __syncthreads();
  {
    const int dig = tid;
    uint32_t run = offs[(int64_t)dig * nblocks + blockIdx.x];
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      const uint32_t c = wc[q][dig];
      wc[q][dig] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t j = base + r * 32 + lane;
    if (j < n) {
      const uint32_t dest = wc[w][d[r]] + lr[r];
      kout[dest] = k[r];
      vout[dest] = v[r];
    }
  }
}

// In-place exclusive scan of a[0..n) by one block of 1024 threads; *total = the sum.
__global__ void __launch_bounds__(kScanThreads) k_scan_single(uint32_t* a, int64_t n, uint32_t* total) {
  __shared__ uint32_t sm[kScanThreads];
  const int t = threadIdx.x;
  const int64_t chunk = (n + kScanThreads - 1) / kScanThreads;
  const int64_t lo = std::min<int64_t>(n, (int64_t)t * chunk);
  const int64_t hi = std::min<int64_t>(n, lo + chunk);
  uint32_t sum = 0;
  for (int64_t i = lo; i < hi; ++i) sum += a[i];
  sm[t] = sum;
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {
    const uint32_t x = t >= off ? sm[t - off] : 0u;
    __syncthreads();
    sm[t] += x;
    __syncthreads();
  }
  uint32_t run = sm[t] - sum;
  if (t == kScanThreads - 1 && total != nullptr) *total = sm[t];
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t x = a[i];
    a[i] = run;
    run += x;
  }
}

__device__ __forceinline__ uint32_t block_exclusive_scan_1024(uint32_t x, uint32_t* warp_tot, uint32_t* block_total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += y;
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    uint32_t t = warp_tot[lane];
    uint32_t ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += y;
    }
    warp_tot[lane] = ti - t;
    if (lane == 31 && block_total) *block_total = ti;
  }
  __syncthreads();
  return warp_tot[w] + inc - x;
}

__global__ void __launch_bounds__(kScanThreads) k_tile_sums(const uint32_t* __restrict__ a, int64_t n,
                                                            uint32_t* __restrict__ sums) {
  __shared__ uint32_t wt[32];
  __shared__ uint32_t tot;
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i)
    if (base + i < n) s += a[base + i];
  block_exclusive_scan_1024(s, wt, &tot);
  __syncthreads();
  if (threadIdx.x == 0) sums[blockIdx.x] = tot;
}

// May run in place (out == a): every thread reads its items before the block scan's
// barriers and writes them after.
__global__ void __launch_bounds__(kScanThreads) k_tile_scan(const uint32_t* a, uint32_t* out, int64_t n,
                                                            const uint32_t* __restrict__ offs) {
  __shared__ uint32_t wt[32];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  uint32_t x[kScanItems];
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    x[i] = base + i < n ? a[base + i] : 0u;
    s += x[i];
  }
  uint32_t run = offs[blockIdx.x] + block_exclusive_scan_1024(s, wt, nullptr);
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    if (base + i < n) out[base + i] = run;
    run += x[i];
  }
}

// ------------------------------------------------------------------------- build kernels

__global__ void k_make_keys(const int32_t* __restrict__ row, const int32_t* __restrict__ col, int64_t nnz, int64_t M,
                            int64_t K, uint64_t* __restrict__ keys, uint32_t* __restrict__ vals, uint32_t* err) {
  bool bad = false;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nnz; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = row[e], c = col[e];
    const bool ok = r >= 0 && r < M && c >= 0 && c < K;
    bad |= !ok;
    keys[e] = ok ? (uint64_t)(r * K + c) : 0ull;
    vals[e] = (uint32_t)e;
  }
  if (bad) atomicOr(err, ERRBIT_OUT_OF_RANGE);
}

__global__ void k_check_dups(const uint64_t* __restrict__ keys, int64_t n, uint32_t* err) {
  bool dup = false;
  for (int64_t i = 1 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dup |= keys[i] == keys[i - 1];
  if (dup) atomicOr(err, ERRBIT_DUPLICATE);
}

template <typename W>
__global__ void k_apply_build(const uint64_t* __restrict__ keys, const uint32_t* __restrict__ src, int64_t nnz, int64_t K,
                              int32_t* __restrict__ row, int32_t* __restrict__ col, const W* __restrict__ vcopy,
                              W* __restrict__ values, const uint32_t* err) {
  if (*err) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nnz; i += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t key = keys[i];
    row[i] = (int32_t)(key / (uint64_t)K);
    col[i] = (int32_t)(key % (uint64_t)K);
    values[i] = vcopy[src[i]];
  }
}

// ptr[r] = number of entries with idx < r, from sorted idx[0..n).
__global__ void k_ptr_from_sorted(const int32_t* __restrict__ idx, int64_t n, int64_t dim, int32_t* __restrict__ ptr,
                                  const uint32_t* err) {
  if (*err) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i <= n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t lo = i == 0 ? 0 : (int64_t)idx[i - 1] + 1;
    const int64_t hi = i == n ? dim : (int64_t)idx[i];
    for (int64_t r = lo; r <= hi; ++r) ptr[r] = (int32_t)i;
  }
}

__global__ void k_csc_keys(const int32_t* __restrict__ col, int64_t nnz, uint64_t* __restrict__ keys,
                           uint32_t* __restrict__ vals, const uint32_t* err) {
  if (*err) return;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nnz; e += (int64_t)gridDim.x * blockDim.x) {
    keys[e] = (uint64_t)col[e];
    vals[e] = (uint32_t)e;
  }
}

__global__ void k_csc_finish(const uint64_t* __restrict__ keys, const uint32_t* __restrict__ src,
                             const int32_t* __restrict__ row, int64_t nnz, int32_t* __restrict__ perm,
                             int32_t* __restrict__ csc_row, int32_t* __restrict__ cols_sorted, const uint32_t* err) {
  if (*err) return;
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < nnz; j += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t e = src[j];
    perm[j] = (int32_t)e;
    csc_row[j] = row[e];
    cols_sorted[j] = (int32_t)keys[j];
  }
}

// part_nnz[p] = floor(p nnz / P); part_idx[p] = last r with ptr[r] <= part_nnz[p] (dim at the end).
__global__ void k_parts(const int32_t* __restrict__ ptr, int64_t dim, int64_t nnz, int P, int32_t* __restrict__ part_nnz,
                        int32_t* __restrict__ part_idx, const uint32_t* err) {
  if (*err) return;
  for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p <= P; p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t a = (p * nnz) / P;
    part_nnz[p] = (int32_t)a;
    if (a >= nnz) {
      part_idx[p] = (int32_t)dim;
      continue;
    }
    int64_t lo = 0, hi = dim + 1;  // first q with ptr[q] > a
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (ptr[mid] <= a) lo = mid + 1; else hi = mid;
    }
    part_idx[p] = (int32_t)(lo - 1);
  }
}

// Last r in [lo, dim] with ptr[r] <= x (the row holding entry x when x < nnz).
__device__ __forceinline__ int64_t row_holding(const int32_t* __restrict__ ptr, int64_t lo, int64_t dim, int64_t x) {
  int64_t hi = dim;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (ptr[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Work descriptor of part p for the product kernels.  The part's nominal range
// [a, b) = [floor(p nnz / P), floor((p+1) nnz / P)) is moved to row boundaries where a
// row shorter than the smallest part crosses it: such a row belongs wholly to the part in
// which it starts (that part extends its end, the next one skips the row's remainder),
// so only rows longer than a part are ever split between CTAs.  desc = {a', b', ra, rb}
// with ra the row holding a' and rb the row holding b' (dim when b' == nnz).
__global__ void k_part_desc(const int32_t* __restrict__ ptr, int64_t dim, int64_t nnz, int P,
                            const int32_t* __restrict__ part_idx, int4* __restrict__ desc, const uint32_t* err) {
  if (*err) return;
  for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < P; p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t a = (p * nnz) / P, b = ((p + 1) * nnz) / P;
    const int64_t lmax = nnz / P;
    int64_t a2 = a, b2 = b;
    if (a < b) {
      const int64_t ra = part_idx[p];
      if (ptr[ra] < a && ptr[ra + 1] - ptr[ra] <= lmax) a2 = ptr[ra + 1];
      const int64_t t = row_holding(ptr, ra, dim - 1, b - 1);
      if (ptr[t + 1] > b && ptr[t + 1] - ptr[t] <= lmax) b2 = ptr[t + 1];
      if (a2 > b2) a2 = b2;
    }
    const int64_t ra2 = a2 < nnz ? row_holding(ptr, 0, dim - 1, a2) : dim;
    const int64_t rb2 = b2 < nnz ? row_holding(ptr, 0, dim - 1, b2) : dim;
    desc[p] = make_int4((int)a2, (int)b2, (int)ra2, (int)rb2);
  }
}

// ------------------------------------------------------------------------- restructure kernels

// 16-bit copy of an index array whose values are known to be < 65536.
__global__ void k_narrow(const int32_t* __restrict__ in, uint16_t* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint16_t)in[i];
}

// dst[old_to_new[e]] = src[e] for the surviving entries of a restructure (dst zeroed first).
template <typename W>
__global__ void k_remap_scatter(const int32_t* __restrict__ old_to_new, int64_t nnz, const W* __restrict__ src,
                                W* __restrict__ dst) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nnz; e += (int64_t)gridDim.x * blockDim.x) {
    const int32_t t = old_to_new[e];
    if (t >= 0 && t < nnz) dst[t] = src[e];
  }
}

template <typename W>
__global__ void k_mag_keys(const W* __restrict__ values, int64_t nnz, uint64_t* __restrict__ keys,
                           uint32_t* __restrict__ vals, uint32_t* err) {
  bool nan = false;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nnz; e += (int64_t)gridDim.x * blockDim.x) {
    uint32_t bits = (uint32_t)values[e];
    if (sizeof(W) == 2) bits <<= 16;  // bf16 -> the float32 with the same value
    const uint32_t mag = bits & 0x7fffffffu;  // |v| as float bits: monotone in |v|, -0 == +0
    nan |= mag > 0x7f800000u;
    keys[e] = mag;
    vals[e] = (uint32_t)e;
  }
  if (nan) atomicOr(err, ERRBIT_INVALID_VALUE);
}

__global__ void k_mark_dropped(const uint32_t* __restrict__ order, int64_t k, uint32_t* __restrict__ dropped) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < k; i += (int64_t)gridDim.x * blockDim.x)
    dropped[order[i]] = 1u;
}

// Output i (0-based) of SplitMix64 seeded with `seed`: the mix of seed + (i + 1) * gamma
// (Steele, Lea and Flood, OOPSLA 2014).
__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1ull) * 0x9e3779b97f4a7c15ull;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ bool position_stored(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                                                uint64_t K, uint64_t pos) {
  const int64_t r = (int64_t)(pos / K);
  const int32_t c = (int32_t)(pos % K);
  int64_t lo = row_ptr[r], hi = row_ptr[r + 1];
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    const int32_t x = col[mid];
    if (x == c) return true;
    if (x < c) lo = mid + 1; else hi = mid;
  }
  return false;
}

// keys[0..nA) = accepted positions (payload 0); keys[nA + j] = draw i0 + j mapped to a
// position, or MK (sorts last, ignored) when the position is in the pre-drop set.
__global__ void k_regrow_fill(uint64_t seed, uint64_t i0, int64_t B, uint64_t MK, uint64_t K,
                              const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col,
                              const uint64_t* __restrict__ grown, int64_t nA, uint64_t* __restrict__ keys,
                              uint32_t* __restrict__ vals) {
  const int64_t n = nA + B;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < n; q += (int64_t)gridDim.x * blockDim.x) {
    if (q < nA) {
      keys[q] = grown[q];
      vals[q] = 0u;
    } else {
      const int64_t j = q - nA;
      const uint64_t u = splitmix64_at(seed, i0 + (uint64_t)j);
      const uint64_t pos = __umul64hi(u, MK);
      keys[q] = position_stored(row_ptr, col, K, pos) ? MK : pos;
      vals[q] = (uint32_t)(j + 1);
    }
  }
}

// After the stable sort by position: the first entry of each run of equal positions is a
// new acceptance when it comes from this batch (payload > 0) and is not the sentinel.
__global__ void k_regrow_keep(const uint64_t* __restrict__ keys, const uint32_t* __restrict__ vals, int64_t n,
                              uint64_t MK, uint32_t* __restrict__ sel, uint64_t* __restrict__ cand) {
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < n; q += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t key = keys[q];
    const uint32_t v = vals[q];
    const bool first = q == 0 || keys[q - 1] != key;
    if (key != MK && first && v > 0u) {
      sel[v - 1] = 1u;
      cand[v - 1] = key;
    }
  }
}

__global__ void k_regrow_take(const uint32_t* __restrict__ sel, const uint32_t* __restrict__ rank,
                              const uint64_t* __restrict__ cand, int64_t B, int64_t need, uint64_t* __restrict__ grown,
                              int64_t nA) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < B; j += (int64_t)gridDim.x * blockDim.x)
    if (sel[j] && (int64_t)rank[j] < need) grown[nA + rank[j]] = cand[j];
}

__global__ void k_merge_keys(const int32_t* __restrict__ row, const int32_t* __restrict__ col, int64_t nnz, uint64_t K,
                             const uint32_t* __restrict__ dropped, const uint64_t* __restrict__ grown, int64_t k,
                             uint64_t MK, uint64_t* __restrict__ keys, uint32_t* __restrict__ vals) {
  const int64_t n = nnz + k;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < n; q += (int64_t)gridDim.x * blockDim.x) {
    if (q < nnz) {
      keys[q] = dropped[q] ? MK : (uint64_t)row[q] * K + (uint64_t)col[q];
      vals[q] = (uint32_t)q;
    } else {
      keys[q] = grown[q - nnz];
      vals[q] = 0x80000000u | (uint32_t)(q - nnz);
    }
  }
}

template <typename W>
__global__ void k_apply_restructure(const uint64_t* __restrict__ keys, const uint32_t* __restrict__ src, int64_t nnz,
                                    uint64_t K, int32_t* __restrict__ row, int32_t* __restrict__ col,
                                    const W* __restrict__ vcopy, W* __restrict__ values, W regrow_bits,
                                    int32_t* __restrict__ old_to_new) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nnz; i += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t key = keys[i];
    row[i] = (int32_t)(key / K);
    col[i] = (int32_t)(key % K);
    const uint32_t s = src[i];
    if (s & 0x80000000u) {
      values[i] = regrow_bits;
    } else {
      values[i] = vcopy[s];
      if (old_to_new != nullptr) old_to_new[s] = (int32_t)i;
    }
  }
}

// ------------------------------------------------------------------------- host helpers

constexpr int kThreads = 256;

cudaError_t fill_u32(uint32_t* p, int64_t n, uint32_t v, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  k_fill_u32<<<grid_for(n, kThreads), kThreads, 0, s>>>(p, n, v);
  return cudaGetLastError();
}

// Sorts (keys0, vals0)[0..n) by key bits [0, nbits).  The result lands in keys0/vals0 or
// keys1/vals1; *alt tells which (true = the "1" buffers).
snk_status radix_sort(snk_layout* L, int64_t n, int nbits, cudaStream_t s, bool* alt) {
  uint64_t* ki = L->keys0;
  uint64_t* ko = L->keys1;
  uint32_t* vi = L->vals0;
  uint32_t* vo = L->vals1;
  if (n > 0) {
    const int nblocks = (int)ceil_div(n, kSortTile);
    const int64_t nh = (int64_t)256 * nblocks;
    const int64_t nt = ceil_div(nh, kScanTile);
    for (int shift = 0; shift < nbits; shift += 8) {
      k_rs_hist<<<nblocks, kSortThreads, 0, s>>>(ki, n, shift, L->hist, nblocks);
      // exclusive scan of the digit-major histogram, in place (tile sums, their scan, tiles)
      k_tile_sums<<<(unsigned)nt, kScanThreads, 0, s>>>(L->hist, nh, L->scan_tmp);
      k_scan_single<<<1, kScanThreads, 0, s>>>(L->scan_tmp, nt, nullptr);
      k_tile_scan<<<(unsigned)nt, kScanThreads, 0, s>>>(L->hist, L->hist, nh, L->scan_tmp);
      k_rs_scatter<<<nblocks, kSortThreads, 0, s>>>(ki, vi, ko, vo, n, shift, L->hist, nblocks);
      std::swap(ki, ko);
      std::swap(vi, vo);
    }
    SNK_CUDA_TRY(cudaGetLastError());
  }
  *alt = ki == L->keys1;
  return SNK_OK;
}

// Exclusive scan of in[0..n) into out[0..n); the total lands in *total_dev.
snk_status scan_u32(snk_layout* L, const uint32_t* in, uint32_t* out, int64_t n, uint32_t* total_dev,
                    cudaStream_t s) {
  const int64_t nt = ceil_div(std::max<int64_t>(n, 1), kScanTile);
  k_tile_sums<<<(unsigned)nt, kScanThreads, 0, s>>>(in, n, L->scan_tmp);
  k_scan_single<<<1, kScanThreads, 0, s>>>(L->scan_tmp, nt, total_dev);
  k_tile_scan<<<(unsigned)nt, kScanThreads, 0, s>>>(in, out, n, L->scan_tmp);
  SNK_CUDA_TRY(cudaGetLastError());
  return SNK_OK;
}

snk_status read_err(snk_layout* L, cudaStream_t s, uint32_t* host_err) {
  SNK_CUDA_TRY(cudaMemcpyAsync(host_err, L->err, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
  SNK_CUDA_TRY(cudaStreamSynchronize(s));
  return SNK_OK;
}

snk_status status_from_err(uint32_t e) {
  if (e & ERRBIT_OUT_OF_RANGE) return SNK_ERR_OUT_OF_RANGE;
  if (e & ERRBIT_DUPLICATE) return SNK_ERR_DUPLICATE;
  if (e & ERRBIT_INVALID_VALUE) return SNK_ERR_INVALID_VALUE;
  return SNK_OK;
}

uint16_t f32_to_bf16_bits_host(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  return (uint16_t)((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

struct Carver {
  uint8_t* base;
  size_t off;
  template <typename T>
  T* take(int64_t count) {
    off = (off + 255) & ~(size_t)255;
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += sizeof(T) * (size_t)std::max<int64_t>(count, 1);
    return p;
  }
};

size_t carve(snk_layout* L, uint8_t* base) {
  Carver c{base, 0};
  const int64_t M = L->M, K = L->K, nnz = L->nnz, P = L->P;
  L->scap = sort_capacity(nnz);
  L->row_ptr = c.take<int32_t>(M + 1);
  L->col_ptr = c.take<int32_t>(K + 1);
  L->csc_row = c.take<int32_t>(nnz);
  L->perm = c.take<int32_t>(nnz);
  L->part_nnz = c.take<int32_t>(P + 1);
  L->part_row = c.take<int32_t>(P + 1);
  L->part_nnz_t = c.take<int32_t>(P + 1);
  L->part_col = c.take<int32_t>(P + 1);
  L->desc_f = c.take<int4>(P);
  L->desc_t = c.take<int4>(P);
  L->carry_tail_f = c.take<float>(P * kCarryCols);
  L->carry_head_f = c.take<float>(P * kCarryCols);
  L->cnt_f = c.take<uint32_t>((int64_t)kMaxTiles * P);
  L->carry_tail_b = c.take<float>(P * kCarryCols);
  L->carry_head_b = c.take<float>(P * kCarryCols);
  L->cnt_b = c.take<uint32_t>((int64_t)kMaxTiles * P);
  L->err = c.take<uint32_t>(64);
  L->keys0 = c.take<uint64_t>(L->scap);
  L->keys1 = c.take<uint64_t>(L->scap);
  L->vals0 = c.take<uint32_t>(L->scap);
  L->vals1 = c.take<uint32_t>(L->scap);
  L->hist = c.take<uint32_t>((int64_t)256 * ceil_div(L->scap, kSortTile));
  L->flags = c.take<uint32_t>(L->scap);
  L->flags2 = c.take<uint32_t>(L->scap);
  L->grown = c.take<uint64_t>(nnz);
  L->vcopy = c.take<uint8_t>(4 * nnz);
  L->scan_tmp = c.take<uint32_t>(ceil_div(L->scap, kScanTile) + ceil_div((int64_t)256 * ceil_div(L->scap, kSortTile), kScanTile) + 64);
  if (index16_possible(M, K)) {
    L->col16 = c.take<uint16_t>(nnz);
    L->csc_row16 = c.take<uint16_t>(nnz);
  } else {
    L->col16 = nullptr;
    L->csc_row16 = nullptr;
  }
  return c.off;
}

}  // namespace

size_t workspace_bytes(int64_t M, int64_t K, int64_t nnz, int32_t P) {
  snk_layout L{};
  L.M = M;
  L.K = K;
  L.nnz = nnz;
  L.P = P;
  return (carve(&L, nullptr) + 256 + 255) / 256 * 256;  // whole 256-byte blocks
}

snk_status layout_carve(snk_layout* L, void* ws, size_t ws_bytes) {
  if (((uintptr_t)ws & 255u) != 0) return SNK_ERR_INVALID_ARG;
  const size_t need = workspace_bytes(L->M, L->K, L->nnz, L->P);
  if (ws_bytes < need) return SNK_ERR_WORKSPACE_TOO_SMALL;
  carve(L, (uint8_t*)ws);
  return SNK_OK;
}

// Row pointers, CSC permutation and partitions from the sorted COO in L->row / L->col.
snk_status derive_format(snk_layout* L, cudaStream_t s) {
  const int64_t nnz = L->nnz;
  k_ptr_from_sorted<<<grid_for(nnz + 1, kThreads), kThreads, 0, s>>>(L->row, nnz, L->M, L->row_ptr, L->err);
  k_csc_keys<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(L->col, nnz, L->keys0, L->vals0, L->err);
  SNK_CUDA_TRY(cudaGetLastError());
  bool alt = false;
  SNK_TRY(radix_sort(L, nnz, bits_for((uint64_t)(L->K - 1)), s, &alt));
  int32_t* cols_sorted = reinterpret_cast<int32_t*>(L->flags);
  k_csc_finish<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(alt ? L->keys1 : L->keys0, alt ? L->vals1 : L->vals0,
                                                            L->row, nnz, L->perm, L->csc_row, cols_sorted, L->err);
  k_ptr_from_sorted<<<grid_for(nnz + 1, kThreads), kThreads, 0, s>>>(cols_sorted, nnz, L->K, L->col_ptr, L->err);
  k_parts<<<grid_for(L->P + 1, kThreads), kThreads, 0, s>>>(L->row_ptr, L->M, nnz, L->P, L->part_nnz, L->part_row,
                                                            L->err);
  k_parts<<<grid_for(L->P + 1, kThreads), kThreads, 0, s>>>(L->col_ptr, L->K, nnz, L->P, L->part_nnz_t, L->part_col,
                                                            L->err);
  k_part_desc<<<grid_for(L->P, kThreads), kThreads, 0, s>>>(L->row_ptr, L->M, nnz, L->P, L->part_row, L->desc_f, L->err);
  k_part_desc<<<grid_for(L->P, kThreads), kThreads, 0, s>>>(L->col_ptr, L->K, nnz, L->P, L->part_col, L->desc_t, L->err);
  SNK_CUDA_TRY(cudaGetLastError());
  if (L->col16 != nullptr) {
    k_narrow<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(L->col, L->col16, nnz);
    k_narrow<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(L->csc_row, L->csc_row16, nnz);
  }
  SNK_CUDA_TRY(cudaGetLastError());
  SNK_CUDA_TRY(fill_u32(L->cnt_f, (int64_t)kMaxTiles * L->P, 0u, s));
  SNK_CUDA_TRY(fill_u32(L->cnt_b, (int64_t)kMaxTiles * L->P, 0u, s));
  return SNK_OK;
}

snk_status build_format(snk_layout* L, void* values, int vbytes, cudaStream_t s) {
  const int64_t nnz = L->nnz;
  SNK_CUDA_TRY(fill_u32(L->err, 64, 0u, s));
  if (nnz > 0) {
    if (vbytes == 4)
      k_copy<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint32_t*)values, (uint32_t*)L->vcopy, nnz);
    else
      k_copy<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint16_t*)values, (uint16_t*)L->vcopy, nnz);
    k_make_keys<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(L->row, L->col, nnz, L->M, L->K, L->keys0, L->vals0, L->err);
    SNK_CUDA_TRY(cudaGetLastError());
    bool alt = false;
    SNK_TRY(radix_sort(L, nnz, bits_for((uint64_t)(L->M * L->K - 1)), s, &alt));
    const uint64_t* ks = alt ? L->keys1 : L->keys0;
    const uint32_t* vs = alt ? L->vals1 : L->vals0;
    k_check_dups<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(ks, nnz, L->err);
    if (vbytes == 4)
      k_apply_build<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(
          ks, vs, nnz, L->K, L->row, L->col, (const uint32_t*)L->vcopy, (uint32_t*)values, L->err);
    else
      k_apply_build<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(
          ks, vs, nnz, L->K, L->row, L->col, (const uint16_t*)L->vcopy, (uint16_t*)values, L->err);
    SNK_CUDA_TRY(cudaGetLastError());
  }
  SNK_TRY(derive_format(L, s));
  uint32_t e = 0;
  SNK_TRY(read_err(L, s, &e));
  return status_from_err(e);
}

snk_status restructure(snk_layout* L, void* values, int64_t k, uint64_t seed, float regrow_value,
                       int32_t* old_to_new, cudaStream_t s) {
  const int64_t nnz = L->nnz;
  const uint64_t MK = (uint64_t)L->M * (uint64_t)L->K;
  const int vbytes = L->dtype == SNK_F32 ? 4 : 2;
  if (k < 0 || k > nnz) return SNK_ERR_INVALID_ARG;
  if ((uint64_t)k > MK - (uint64_t)nnz) return SNK_ERR_NO_ROOM;
  SNK_CUDA_TRY(fill_u32(L->err, 64, 0u, s));
  // NaN check always runs (it is part of the contract even for k == 0).
  if (vbytes == 4)
    k_mag_keys<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint32_t*)values, nnz, L->keys0, L->vals0, L->err);
  else
    k_mag_keys<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint16_t*)values, nnz, L->keys0, L->vals0, L->err);
  SNK_CUDA_TRY(cudaGetLastError());
  uint32_t e = 0;
  SNK_TRY(read_err(L, s, &e));
  if (e) return status_from_err(e);
  if (k == 0) {
    if (old_to_new != nullptr && nnz > 0) {
      k_iota_i32<<<grid_for(nnz, kThreads), kThreads, 0, s>>>(old_to_new, nnz);
      SNK_CUDA_TRY(cudaGetLastError());
      SNK_CUDA_TRY(cudaStreamSynchronize(s));
    }
    return SNK_OK;
  }

  // 1. drop: the k smallest by (|v|, position) -- a stable sort of |v| over the sorted COO.
  bool alt = false;
  SNK_TRY(radix_sort(L, nnz, 31, s, &alt));
  uint32_t* dropped = L->flags;
  SNK_CUDA_TRY(fill_u32(dropped, nnz, 0u, s));
  k_mark_dropped<<<grid_for(k, kThreads), kThreads, 0, s>>>(alt ? L->vals1 : L->vals0, k, dropped);
  SNK_CUDA_TRY(cudaGetLastError());

  // 2. regrowth in rounds of B draws; accepted positions accumulate in L->grown[0..nA).
  const int nbits = bits_for(MK);
  int64_t nA = 0;
  uint64_t i0 = 0;
  const uint64_t kMaxDraws = 1ull << 32;
  uint32_t* total_dev = L->err + 1;
  while (nA < k) {
    int64_t B = L->scap - nA;
    if (i0 >= kMaxDraws) return SNK_ERR_TIMEOUT;
    if ((uint64_t)B > kMaxDraws - i0) B = (int64_t)(kMaxDraws - i0);
    const int64_t n = nA + B;
    k_regrow_fill<<<grid_for(n, kThreads), kThreads, 0, s>>>(seed, i0, B, MK, (uint64_t)L->K, L->row_ptr, L->col,
                                                             L->grown, nA, L->keys0, L->vals0);
    SNK_CUDA_TRY(cudaGetLastError());
    SNK_TRY(radix_sort(L, n, nbits, s, &alt));
    const uint64_t* ks = alt ? L->keys1 : L->keys0;
    const uint32_t* vs = alt ? L->vals1 : L->vals0;
    uint64_t* cand = alt ? L->keys0 : L->keys1;
    uint32_t* rank = alt ? L->vals0 : L->vals1;
    uint32_t* sel = L->flags2;
    SNK_CUDA_TRY(fill_u32(sel, B, 0u, s));
    k_regrow_keep<<<grid_for(n, kThreads), kThreads, 0, s>>>(ks, vs, n, MK, sel, cand);
    SNK_CUDA_TRY(cudaGetLastError());
    SNK_TRY(scan_u32(L, sel, rank, B, total_dev, s));
    const int64_t need = k - nA;
    k_regrow_take<<<grid_for(B, kThreads), kThreads, 0, s>>>(sel, rank, cand, B, need, L->grown, nA);
    SNK_CUDA_TRY(cudaGetLastError());
    uint32_t total = 0;
    SNK_CUDA_TRY(cudaMemcpyAsync(&total, total_dev, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
    SNK_CUDA_TRY(cudaStreamSynchronize(s));
    nA += std::min<int64_t>((int64_t)total, need);
    i0 += (uint64_t)B;
  }

  // 3. merge survivors and regrown positions, sort by position, rewrite the COO.
  if (vbytes == 4)
    k_copy<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint32_t*)values, (uint32_t*)L->vcopy, nnz);
  else
    k_copy<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>((const uint16_t*)values, (uint16_t*)L->vcopy, nnz);
  k_merge_keys<<<grid_for(nnz + k, kThreads), kThreads, 0, s>>>(L->row, L->col, nnz, (uint64_t)L->K, dropped, L->grown,
                                                                k, MK, L->keys0, L->vals0);
  SNK_CUDA_TRY(cudaGetLastError());
  SNK_TRY(radix_sort(L, nnz + k, nbits, s, &alt));
  if (old_to_new != nullptr) SNK_CUDA_TRY(fill_u32((uint32_t*)old_to_new, nnz, 0xffffffffu, s));
  const uint64_t* ks = alt ? L->keys1 : L->keys0;
  const uint32_t* vs = alt ? L->vals1 : L->vals0;
  if (vbytes == 4) {
    uint32_t rb;
    memcpy(&rb, &regrow_value, 4);
    k_apply_restructure<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(
        ks, vs, nnz, (uint64_t)L->K, L->row, L->col, (const uint32_t*)L->vcopy, (uint32_t*)values, rb, old_to_new);
  } else {
    const uint16_t rb = f32_to_bf16_bits_host(regrow_value);
    k_apply_restructure<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(
        ks, vs, nnz, (uint64_t)L->K, L->row, L->col, (const uint16_t*)L->vcopy, (uint16_t*)values, rb, old_to_new);
  }
  SNK_CUDA_TRY(cudaGetLastError());

  // 4. rebuild the derived arrays.
  SNK_TRY(derive_format(L, s));
  SNK_TRY(read_err(L, s, &e));
  return status_from_err(e);
}

snk_status remap_entries(const int32_t* old_to_new, int64_t nnz, const void* src, void* dst, int elem_bytes,
                         cudaStream_t s) {
  if (nnz == 0) return SNK_OK;
  SNK_CUDA_TRY(cudaMemsetAsync(dst, 0, (size_t)nnz * (size_t)elem_bytes, s));
  if (elem_bytes == 4)
    k_remap_scatter<uint32_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(old_to_new, nnz, (const uint32_t*)src,
                                                                           (uint32_t*)dst);
  else
    k_remap_scatter<uint16_t><<<grid_for(nnz, kThreads), kThreads, 0, s>>>(old_to_new, nnz, (const uint16_t*)src,
                                                                           (uint16_t*)dst);
  SNK_CUDA_TRY(cudaGetLastError());
  return SNK_OK;
}

}  // namespace snk
