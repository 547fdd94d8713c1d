/*
 * CPU oracle for the ragged MoE grouped GEMM: plain fp64 loops over bf16 inputs.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg do. It shares no
 * code, header, table or helper with the CUDA library.
 *
 * What it computes (each is the plain definition, written out):
 *   forward  out[r,n] = sum_k A[r,k] * W[e,k,n]        for every row r of group e
 *            (torch._grouped_mm(x, w, offs) in PyTorch issue 152668, "Easy repro scenario")
 *   dgrad    dX[r,k]  = sum_n dY[r,n] * W[e,k,n]       (the grad of x in the same repro's
 *            o.backward; TransformerEngine PR 3542, "Changes": forward, dgrad, wgrad)
 *   wgrad    dW[e,k,n]= sum_{r in group e} A[r,k] * dY[r,n]   ("overwrite wgrad",
 *            TransformerEngine PR 3542, "Changes"); an empty group gives exactly 0
 *   masked   out[e,r,n] = sum_k A[e,r,k] * W[e,k,n]    for r < masked_m[e]
 *            (sglang PR 32385, "Fix": masked_m excludes the inactive rows from the GEMM)
 *
 * Groups come from cumulative END offsets offs[E] (no leading zero): group e covers rows
 * [offs[e-1], offs[e]) with offs[-1] = 0 (the repro's (8,16,32,40) for 4 experts over 48
 * rows). Offsets the pages leave undefined (decreasing, negative, past the buffer) are read
 * with one clamp rule: t'_{-1} = 0, t'_e = clamp(offs[e], t'_{e-1}, rows_alloc).
 * masked_m is clamped to [0, mmax].
 *
 * Every bf16 value is widened exactly to double; each product of two bf16 values is exact
 * in double; the sums run in index order in double. The loop order (row, reduction index,
 * output column) keeps, for every output element, the terms in increasing reduction index,
 * which is the definition's order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t h) {
  uint32_t bits = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

int gg_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Effective bounds of every group; returns 1 when the clamp changed any offset. */
int gg_oracle_group_bounds(const int32_t* offs, int32_t E, int64_t rows_alloc,
                           int64_t* starts, int64_t* ends) {
  int bad = 0;
  int64_t prev = 0;
  for (int32_t e = 0; e < E; ++e) {
    int64_t t = offs[e];
    if (t < prev) t = prev;
    if (t > rows_alloc) t = rows_alloc;
    if (t != (int64_t)offs[e]) bad = 1;
    starts[e] = prev;
    ends[e] = t;
    prev = t;
  }
  return bad;
}

/* Group of row r under the effective bounds, or -1 when r is in no group. */
static int32_t group_of_row(const int64_t* starts, const int64_t* ends, int32_t E, int64_t r) {
  for (int32_t e = 0; e < E; ++e)
    if (r >= starts[e] && r < ends[e]) return e;
  return -1;
}

/* Forward on a list of rows: out[i, n] for row rows[i]; NaN rows for rows in no group. */
void gg_oracle_forward_rows(const uint16_t* A, const uint16_t* W, const int32_t* offs,
                            int32_t E, int64_t rows_alloc, int64_t K, int64_t N,
                            const int64_t* rows, int64_t nrows, double* out,
                            int32_t* group_of, int threads) {
  int64_t* starts = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  int64_t* ends = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  gg_oracle_group_bounds(offs, E, rows_alloc, starts, ends);
#pragma omp parallel for num_threads(threads) schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t r = rows[i];
    const int32_t e = group_of_row(starts, ends, E, r);
    double* o = out + i * N;
    group_of[i] = e;
    if (e < 0) {
      for (int64_t n = 0; n < N; ++n) o[n] = NAN;
      continue;
    }
    for (int64_t n = 0; n < N; ++n) o[n] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      const double a = bf16_to_double(A[r * K + k]);
      const uint16_t* w = W + ((int64_t)e * K + k) * N;
      for (int64_t n = 0; n < N; ++n) o[n] += a * bf16_to_double(w[n]);
    }
  }
  free(starts);
  free(ends);
}

/* Dgrad on a list of rows: dX[i, k] = sum_n dY[r,n] * W[e,k,n]. */
void gg_oracle_dgrad_rows(const uint16_t* dY, const uint16_t* W, const int32_t* offs,
                          int32_t E, int64_t rows_alloc, int64_t K, int64_t N,
                          const int64_t* rows, int64_t nrows, double* out,
                          int32_t* group_of, int threads) {
  int64_t* starts = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  int64_t* ends = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  gg_oracle_group_bounds(offs, E, rows_alloc, starts, ends);
#pragma omp parallel for num_threads(threads) schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t r = rows[i];
    const int32_t e = group_of_row(starts, ends, E, r);
    double* o = out + i * K;
    group_of[i] = e;
    if (e < 0) {
      for (int64_t k = 0; k < K; ++k) o[k] = NAN;
      continue;
    }
    for (int64_t k = 0; k < K; ++k) {
      const uint16_t* w = W + ((int64_t)e * K + k) * N;
      const uint16_t* g = dY + r * N;
      double s = 0.0;
      for (int64_t n = 0; n < N; ++n) s += bf16_to_double(g[n]) * bf16_to_double(w[n]);
      o[k] = s;
    }
  }
  free(starts);
  free(ends);
}

/* Wgrad on a list of reduction-output rows ks (rows of dW[e], i.e. K indices):
   dW[e, j, n] = sum_{r in group e} A[r, ks[j]] * dY[r, n]; exactly 0 for an empty group. */
void gg_oracle_wgrad_krows(const uint16_t* A, const uint16_t* dY, const int32_t* offs,
                           int32_t E, int64_t rows_alloc, int64_t K, int64_t N,
                           const int64_t* ks, int64_t nk, double* dW, int threads) {
  int64_t* starts = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  int64_t* ends = (int64_t*)malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  gg_oracle_group_bounds(offs, E, rows_alloc, starts, ends);
  const int64_t jobs = (int64_t)E * nk;
#pragma omp parallel for num_threads(threads) schedule(dynamic, 1)
  for (int64_t job = 0; job < jobs; ++job) {
    const int32_t e = (int32_t)(job / nk);
    const int64_t j = job % nk;
    const int64_t k = ks[j];
    double* o = dW + job * N;
    for (int64_t n = 0; n < N; ++n) o[n] = 0.0;
    for (int64_t r = starts[e]; r < ends[e]; ++r) {
      const double a = bf16_to_double(A[r * K + k]);
      const uint16_t* g = dY + r * N;
      for (int64_t n = 0; n < N; ++n) o[n] += a * bf16_to_double(g[n]);
    }
  }
  free(starts);
  free(ends);
}

/* Masked forward on a list of flat rows (e * mmax + r): out[i, n] for active rows,
   NaN rows and active[i] = 0 for rows r >= clamp(masked_m[e], 0, mmax).
   Returns 1 when any masked_m lay outside [0, mmax]. */
int gg_oracle_masked_forward_rows(const uint16_t* A, const uint16_t* W,
                                  const int32_t* masked_m, int32_t E, int64_t mmax,
                                  int64_t K, int64_t N, const int64_t* rows, int64_t nrows,
                                  double* out, int32_t* active, int threads) {
  int bad = 0;
  for (int32_t e = 0; e < E; ++e)
    if (masked_m[e] < 0 || masked_m[e] > mmax) bad = 1;
#pragma omp parallel for num_threads(threads) schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    const int64_t fr = rows[i];
    const int32_t e = (int32_t)(fr / mmax);
    const int64_t r = fr % mmax;
    int64_t m = masked_m[e];
    if (m < 0) m = 0;
    if (m > mmax) m = mmax;
    double* o = out + i * N;
    active[i] = r < m;
    if (r >= m) {
      for (int64_t n = 0; n < N; ++n) o[n] = NAN;
      continue;
    }
    for (int64_t n = 0; n < N; ++n) o[n] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      const double a = bf16_to_double(A[fr * K + k]);
      const uint16_t* w = W + ((int64_t)e * K + k) * N;
      for (int64_t n = 0; n < N; ++n) o[n] += a * bf16_to_double(w[n]);
    }
  }
  return bad;
}

/* Round a double to the nearest bf16 (ties to even), directly from the double so that no
   intermediate float rounding happens. Overflow gives +-inf, NaN gives a quiet NaN. */
uint16_t gg_oracle_round_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  const uint16_t sign = signbit(x) ? 0x8000 : 0;
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  double q;
  if (ax < ldexp(1.0, -126)) {
    /* subnormal range of bf16: spacing 2^-133 */
    q = nearbyint(ldexp(ax, 133));
    q = ldexp(q, -133);
  } else {
    int ex;
    double m = frexp(ax, &ex); /* ax = m * 2^ex, 0.5 <= m < 1 */
    q = ldexp(nearbyint(ldexp(m, 8)), ex - 8); /* 8 significant bits */
  }
  if (q >= ldexp(1.0, 128)) return sign | 0x7F80;
  float f = (float)q; /* exact: q has at most 8 significant bits and is in float range */
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  return (uint16_t)(sign | ((bits >> 16) & 0x7FFF));
}

void gg_oracle_round_bf16_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = gg_oracle_round_bf16(x[i]);
}
