/*
 * oracle.c -- plain, slow, single-threaded CPU reference of the truly-sparse layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file or the library built from it: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no source, header, table or helper with the CUDA
 * library under sparse_spmm_b200/csrc.
 *
 * What it computes (source: "Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural
 * Networks on GPU", arXiv 2610.04093, Abstract: a layer that "stores and computes only
 * non-zero connections" in COO format, backpropagates "entirely in the sparse paradigm"
 * and offers an API for "restructuring connections"):
 *
 *   orc_build        O1-O4: validate, sort the COO by (row, col), row pointers, the CSC
 *                    permutation, nnz-balanced partitions.
 *   orc_forward      O5: Y[r,n]  = sum over entries e with row_e = r of v_e * X[col_e, n]
 *   orc_backward_input
 *                    O6: dX[c,n] = sum over entries e with col_e = c of v_e * dY[row_e, n]
 *   orc_backward_weight
 *                    O7: dW[e]   = sum over n of dY[row_e, n] * X[col_e, n]
 *   orc_restructure  O8: magnitude drop of k entries, random regrowth of k positions drawn
 *                    from a SplitMix64 stream, rebuild of the sorted COO.
 *   orc_conv3x3      a 3x3 convolution (stride 1, zero padding 1, no bias) of a
 *                    channel-major input by a sparse kernel whose column index is
 *                    ci*9 + kh*3 + kw ("SparseRT", arXiv 2008.11849, Abstract: sparse
 *                    1x1 and 3x3 convolutions), straight from the definition.
 *   orc_im2col3x3    the patch matrix of that convolution, element bits copied.
 *
 * Every product is accumulated in double.  Each fp routine also returns, per output,
 * the sum of absolute values of its terms (A), which scales the parity tolerance.
 * The pages fix no drop rule, generator, tie-break or partition formula; the readings
 * taken here are stated at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum {
  ORC_OK = 0,
  ORC_INVALID_ARG = 1,
  ORC_OUT_OF_RANGE = 2,
  ORC_DUPLICATE = 3,
  ORC_INVALID_VALUE = 6,
  ORC_NO_ROOM = 7
};

/* ------------------------------------------------------------------ sorting keys */

typedef struct {
  int64_t key; /* primary */
  int64_t tie; /* secondary */
  int64_t src; /* payload */
} orc_item;

static int orc_item_cmp(const void* pa, const void* pb) {
  const orc_item* a = (const orc_item*)pa;
  const orc_item* b = (const orc_item*)pb;
  if (a->key != b->key) return a->key < b->key ? -1 : 1;
  if (a->tie != b->tie) return a->tie < b->tie ? -1 : 1;
  return 0;
}

typedef struct {
  double mag;  /* |v|, exact */
  int64_t lin; /* row * K + col */
  int64_t src;
} orc_mag_item;

static int orc_mag_cmp(const void* pa, const void* pb) {
  const orc_mag_item* a = (const orc_mag_item*)pa;
  const orc_mag_item* b = (const orc_mag_item*)pb;
  if (a->mag != b->mag) return a->mag < b->mag ? -1 : 1;
  if (a->lin != b->lin) return a->lin < b->lin ? -1 : 1;
  return 0;
}

/* ------------------------------------------------------------------ O4: partitions */

/*
 * Reading of "nnz-balanced work partitions": P parts, part p covering the entries
 * [floor(p*nnz/P), floor((p+1)*nnz/P)) of the sorted order, so part sizes differ by at
 * most one.  part_idx[p] is the row (or column, for the CSC copy) that holds the first
 * entry of part p, i.e. the last r with ptr[r] <= part_nnz[p]; it is `dim` when
 * part_nnz[p] == nnz.  P is clamped to max(nnz, 1) so that no part is empty.
 */
static void orc_partitions(const int32_t* ptr, int64_t dim, int64_t nnz, int32_t P,
                           int32_t* part_nnz, int32_t* part_idx) {
  for (int64_t p = 0; p <= P; ++p) {
    int64_t a = (p * nnz) / P;
    part_nnz[p] = (int32_t)a;
    if (a >= nnz) {
      part_idx[p] = (int32_t)dim;
      continue;
    }
    int64_t r = 0;
    for (int64_t q = 0; q <= dim; ++q) /* plain scan: last q with ptr[q] <= a */
      if (ptr[q] <= a) r = q;
    part_idx[p] = (int32_t)r;
  }
}

int32_t orc_effective_parts(int64_t nnz, int32_t P) {
  int64_t cap = nnz > 0 ? nnz : 1;
  return (int32_t)((int64_t)P < cap ? (int64_t)P : cap);
}

/* ------------------------------------------------------------------ O1-O4: build */

/*
 * O1: every row must lie in [0, M) and every col in [0, K) (else OUT_OF_RANGE); no
 * (row, col) may appear twice (else DUPLICATE: a weight matrix holds one value per
 * position).  The entries are sorted by (row, col); since the keys are unique the
 * sorted order is unique.  Values travel with their entries bit for bit.
 * O2: row_ptr[r] = number of entries with row < r.
 * O3: perm lists the sorted-COO indices in (col, row) order; col_ptr[c] = number of
 * entries with col < c; csc_row[j] = row[perm[j]].
 * O4: see orc_partitions.  Outputs are written only when the status is ORC_OK.
 */
int orc_build(int64_t M, int64_t K, int64_t nnz, const int32_t* row_in, const int32_t* col_in,
              const uint8_t* val_in, int vbytes, int32_t P_req, int32_t* row, int32_t* col,
              uint8_t* val, int32_t* row_ptr, int32_t* perm, int32_t* col_ptr, int32_t* csc_row,
              int32_t* P_eff, int32_t* part_nnz, int32_t* part_row, int32_t* part_nnz_t,
              int32_t* part_col) {
  if (M < 1 || K < 1 || nnz < 0 || P_req < 1 || (vbytes != 2 && vbytes != 4)) return ORC_INVALID_ARG;
  for (int64_t e = 0; e < nnz; ++e)
    if (row_in[e] < 0 || row_in[e] >= M || col_in[e] < 0 || col_in[e] >= K) return ORC_OUT_OF_RANGE;

  orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(nnz > 0 ? nnz : 1));
  for (int64_t e = 0; e < nnz; ++e) {
    it[e].key = row_in[e];
    it[e].tie = col_in[e];
    it[e].src = e;
  }
  qsort(it, (size_t)nnz, sizeof(orc_item), orc_item_cmp);
  for (int64_t e = 1; e < nnz; ++e)
    if (it[e].key == it[e - 1].key && it[e].tie == it[e - 1].tie) {
      free(it);
      return ORC_DUPLICATE;
    }
  for (int64_t e = 0; e < nnz; ++e) {
    row[e] = (int32_t)it[e].key;
    col[e] = (int32_t)it[e].tie;
    memcpy(val + e * vbytes, val_in + it[e].src * vbytes, (size_t)vbytes);
  }

  /* O2 */
  for (int64_t r = 0; r <= M; ++r) row_ptr[r] = 0;
  for (int64_t e = 0; e < nnz; ++e) row_ptr[row[e] + 1] += 1;
  for (int64_t r = 0; r < M; ++r) row_ptr[r + 1] += row_ptr[r];

  /* O3 */
  for (int64_t e = 0; e < nnz; ++e) {
    it[e].key = col[e];
    it[e].tie = row[e];
    it[e].src = e;
  }
  qsort(it, (size_t)nnz, sizeof(orc_item), orc_item_cmp);
  for (int64_t j = 0; j < nnz; ++j) {
    perm[j] = (int32_t)it[j].src;
    csc_row[j] = row[perm[j]];
  }
  for (int64_t c = 0; c <= K; ++c) col_ptr[c] = 0;
  for (int64_t e = 0; e < nnz; ++e) col_ptr[col[e] + 1] += 1;
  for (int64_t c = 0; c < K; ++c) col_ptr[c + 1] += col_ptr[c];
  free(it);

  /* O4 */
  int32_t P = orc_effective_parts(nnz, P_req);
  *P_eff = P;
  orc_partitions(row_ptr, M, nnz, P, part_nnz, part_row);
  orc_partitions(col_ptr, K, nnz, P, part_nnz_t, part_col);
  return ORC_OK;
}

/* ------------------------------------------------------------------ O5-O7: products */

/* O5: Y = W X with W given by its entries; X is K x N and Y is M x N, both row-major. */
void orc_forward(int64_t M, int64_t K, int64_t nnz, const int32_t* row, const int32_t* col,
                 const double* val, const double* X, int64_t N, double* Y, double* A) {
  (void)K;
  for (int64_t i = 0; i < M * N; ++i) {
    Y[i] = 0.0;
    A[i] = 0.0;
  }
  for (int64_t e = 0; e < nnz; ++e)
    for (int64_t n = 0; n < N; ++n) {
      double t = val[e] * X[(int64_t)col[e] * N + n];
      Y[(int64_t)row[e] * N + n] += t;
      A[(int64_t)row[e] * N + n] += fabs(t);
    }
}

/* O6: dX = W^T dY; dY is M x N and dX is K x N, both row-major. */
void orc_backward_input(int64_t M, int64_t K, int64_t nnz, const int32_t* row, const int32_t* col,
                        const double* val, const double* dY, int64_t N, double* dX, double* A) {
  (void)M;
  for (int64_t i = 0; i < K * N; ++i) {
    dX[i] = 0.0;
    A[i] = 0.0;
  }
  for (int64_t e = 0; e < nnz; ++e)
    for (int64_t n = 0; n < N; ++n) {
      double t = val[e] * dY[(int64_t)row[e] * N + n];
      dX[(int64_t)col[e] * N + n] += t;
      A[(int64_t)col[e] * N + n] += fabs(t);
    }
}

/* O7: dW[e] = (dY X^T)[row_e, col_e], one value per stored entry, in the given order. */
void orc_backward_weight(int64_t nnz, const int32_t* row, const int32_t* col, const double* dY,
                         const double* X, int64_t N, double* dW, double* A) {
  for (int64_t e = 0; e < nnz; ++e) {
    double s = 0.0, a = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      double t = dY[(int64_t)row[e] * N + n] * X[(int64_t)col[e] * N + n];
      s += t;
      a += fabs(t);
    }
    dW[e] = s;
    A[e] = a;
  }
}

/* ------------------------------------------------------------------ O8: restructure */

/*
 * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014; the 64-bit finaliser with shifts 30/27/31 is Stafford's "Mix13"): the state
 * advances by the golden-ratio increment and each output is the finaliser of the state.
 * Output i (i = 0, 1, ...) is therefore mix(seed + (i + 1) * 0x9e3779b97f4a7c15).
 */
static uint64_t orc_sm64_next(uint64_t* state) {
  uint64_t z = (*state += 0x9e3779b97f4a7c15ULL);
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

void orc_splitmix64(uint64_t seed, int64_t n, uint64_t* out) {
  uint64_t s = seed;
  for (int64_t i = 0; i < n; ++i) out[i] = orc_sm64_next(&s);
}

/* float -> bfloat16 bits, round to nearest even (NaN kept quiet). */
static uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/*
 * Reading of "restructuring connections" (the pages give no drop or grow rule):
 *  1. Drop the k entries with the smallest |v| (exact widening; -0 equals +0); ties go
 *     to the smaller linear index row*K + col.  A NaN value is INVALID_VALUE.
 *  2. Regrow: walk the SplitMix64 stream seeded with `seed`; draw i maps to the position
 *     c_i = floor(u_i * (M*K) / 2^64) (a 128-bit product, Lemire's multiply-shift).  A
 *     position is accepted when it is not in the PRE-drop set and was not accepted
 *     before; the walk stops at k acceptances.  k > M*K - nnz is NO_ROOM.
 *  3. Regrown entries take `regrow_value` rounded to the value type (RNE for bf16);
 *     survivors keep their value bits.
 *  4. The survivors and the regrown positions are sorted by (row, col) again;
 *     old_to_new[e] is the new index of surviving entry e, -1 when e was dropped.
 * Input: the sorted COO of a valid layout.  *draws_out reports how many draws were used.
 */
int orc_restructure(int64_t M, int64_t K, int64_t nnz, const int32_t* row, const int32_t* col,
                    const uint8_t* val_raw, const double* val_f64, int vbytes, int64_t k,
                    uint64_t seed, double regrow_value, int32_t* row_out, int32_t* col_out,
                    uint8_t* val_out, int32_t* old_to_new, int64_t* draws_out) {
  if (vbytes != 2 && vbytes != 4) return ORC_INVALID_ARG;
  if (k < 0 || k > nnz) return ORC_INVALID_ARG;
  for (int64_t e = 0; e < nnz; ++e)
    if (isnan(val_f64[e])) return ORC_INVALID_VALUE;
  int64_t MK = M * K;
  if (k > MK - nnz) return ORC_NO_ROOM;

  /* 1. magnitude ranking by (|v|, linear index) */
  orc_mag_item* mi = (orc_mag_item*)malloc(sizeof(orc_mag_item) * (size_t)(nnz > 0 ? nnz : 1));
  for (int64_t e = 0; e < nnz; ++e) {
    mi[e].mag = fabs(val_f64[e]);
    mi[e].lin = (int64_t)row[e] * K + col[e];
    mi[e].src = e;
  }
  qsort(mi, (size_t)nnz, sizeof(orc_mag_item), orc_mag_cmp);
  unsigned char* dropped = (unsigned char*)calloc((size_t)(nnz > 0 ? nnz : 1), 1);
  for (int64_t i = 0; i < k; ++i) dropped[mi[i].src] = 1;
  free(mi);
  orc_item* it = (orc_item*)malloc(sizeof(orc_item) * (size_t)(nnz > 0 ? nnz : 1));

  /* 2. regrowth: a bitmap over all M*K positions marks the pre-drop set and acceptances */
  unsigned char* taken = (unsigned char*)calloc((size_t)(MK / 8 + 1), 1);
  for (int64_t e = 0; e < nnz; ++e) {
    int64_t lin = (int64_t)row[e] * K + col[e];
    taken[lin >> 3] |= (unsigned char)(1u << (lin & 7));
  }
  int64_t* grown = (int64_t*)malloc(sizeof(int64_t) * (size_t)(k > 0 ? k : 1));
  int64_t accepted = 0, draws = 0;
  uint64_t state = seed;
  while (accepted < k) {
    uint64_t u = orc_sm64_next(&state);
    ++draws;
    int64_t c = (int64_t)(((unsigned __int128)u * (unsigned __int128)(uint64_t)MK) >> 64);
    if (taken[c >> 3] & (1u << (c & 7))) continue;
    taken[c >> 3] |= (unsigned char)(1u << (c & 7));
    grown[accepted++] = c;
  }
  free(taken);
  *draws_out = draws;

  /* 3. new value bits for regrown entries */
  uint8_t rv[4];
  if (vbytes == 4) {
    float f = (float)regrow_value;
    memcpy(rv, &f, 4);
  } else {
    uint16_t b = orc_f32_to_bf16((float)regrow_value);
    memcpy(rv, &b, 2);
  }

  /* 4. merge and sort by (row, col) */
  int64_t n2 = 0;
  for (int64_t e = 0; e < nnz; ++e) {
    old_to_new[e] = -1;
    if (dropped[e]) continue;
    it[n2].key = (int64_t)row[e] * K + col[e];
    it[n2].tie = 0;
    it[n2].src = e;
    ++n2;
  }
  for (int64_t j = 0; j < k; ++j) {
    it[n2].key = grown[j];
    it[n2].tie = 0;
    it[n2].src = -1 - j;
    ++n2;
  }
  qsort(it, (size_t)n2, sizeof(orc_item), orc_item_cmp);
  for (int64_t i = 0; i < n2; ++i) {
    row_out[i] = (int32_t)(it[i].key / K);
    col_out[i] = (int32_t)(it[i].key % K);
    if (it[i].src >= 0) {
      memcpy(val_out + i * vbytes, val_raw + it[i].src * vbytes, (size_t)vbytes);
      old_to_new[it[i].src] = (int32_t)i;
    } else {
      memcpy(val_out + i * vbytes, rv, (size_t)vbytes);
    }
  }
  free(grown);
  free(dropped);
  free(it);
  return ORC_OK;
}

/* ------------------------------------------------------------------ 3x3 convolution */

/* Y[co][n][h][w] = sum over entries (co, c = ci*9 + kh*3 + kw) of v * X[ci][n][h+kh-1][w+kw-1],
 * terms outside the image being zero.  X: C x Nb x H x W, Y: Co x Nb x H x W, row-major. */
void orc_conv3x3(int64_t Co, int64_t C, int64_t Nb, int64_t H, int64_t W, int64_t nnz, const int32_t* row,
                 const int32_t* col, const double* val, const double* X, double* Y, double* A) {
  (void)C;
  const int64_t P = Nb * H * W;
  for (int64_t i = 0; i < Co * P; ++i) {
    Y[i] = 0.0;
    A[i] = 0.0;
  }
  for (int64_t e = 0; e < nnz; ++e) {
    const int64_t co = row[e], ci = col[e] / 9, kh = (col[e] / 3) % 3, kw = col[e] % 3;
    for (int64_t n = 0; n < Nb; ++n)
      for (int64_t h = 0; h < H; ++h)
        for (int64_t w = 0; w < W; ++w) {
          const int64_t hs = h + kh - 1, ws = w + kw - 1;
          if (hs < 0 || hs >= H || ws < 0 || ws >= W) continue;
          const double t = val[e] * X[((ci * Nb + n) * H + hs) * W + ws];
          Y[co * P + (n * H + h) * W + w] += t;
          A[co * P + (n * H + h) * W + w] += fabs(t);
        }
  }
}

/* Patch matrix of the convolution above: out[(ci*9 + kh*3 + kw)][(n*H + h)*W + w] =
 * X[ci][n][h+kh-1][w+kw-1], or all-zero bits outside the image.  Elements of `elem`
 * bytes are copied bit for bit; out has row stride ld (elements). */
void orc_im2col3x3(int64_t C, int64_t Nb, int64_t H, int64_t W, int elem, const void* X, void* out, int64_t ld) {
  const int64_t P = Nb * H * W;
  const unsigned char* x = (const unsigned char*)X;
  unsigned char* o = (unsigned char*)out;
  for (int64_t ci = 0; ci < C; ++ci)
    for (int64_t k = 0; k < 9; ++k) {
      const int64_t kh = k / 3, kw = k % 3, r = ci * 9 + k;
      for (int64_t n = 0; n < Nb; ++n)
        for (int64_t h = 0; h < H; ++h)
          for (int64_t w = 0; w < W; ++w) {
            const int64_t hs = h + kh - 1, ws = w + kw - 1, j = (n * H + h) * W + w;
            unsigned char* dst = o + (r * ld + j) * elem;
            if (hs < 0 || hs >= H || ws < 0 || ws >= W)
              memset(dst, 0, (size_t)elem);
            else
              memcpy(dst, x + (((ci * Nb + n) * H + hs) * W + ws) * elem, (size_t)elem);
          }
    }
  (void)P;
}
