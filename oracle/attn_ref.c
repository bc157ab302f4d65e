/*
 * Oracle for the dense attention forward pass -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this file's library.  The product (the CUDA path) never calls it and
 * shares no code with it.
 *
 * What it computes (page "lecompute.fr/kernel-perf/flashattention-4-limites-
 * calcul-matriciel", section "Entre deux multiplications il faut fabriquer
 * les poids"): queries Q are compared with keys K by a first matrix product,
 * which gives scores; a softmax turns each row of scores into positive
 * weights that sum to one; a second product mixes the values V with those
 * weights.  The same page's section "Le FP4 ajoute un compromis numerique"
 * restricts each position, under the causal mask, to the positions the mask
 * allows; the plain reading used here is "key j is visible to query i iff
 * j <= i" (queries and keys have the same length N, so top-left and
 * bottom-right alignment coincide).
 *
 * The tiled / online-softmax method the pages describe reorders this sum but
 * reaches the same result (section "Entre deux multiplications...": tiling
 * accumulates the result instead of storing the score matrix, it does not
 * remove any comparison).  So this oracle is the plain definition, written
 * out row by row in fp64, with no blocking and no running rescale:
 *
 *   s_j    = scale * sum_c q[i,c] * k[j,c]              j in J(i)
 *   m      = max_j s_j
 *   l      = sum_j exp(s_j - m)
 *   O[i,c] = sum_j exp(s_j - m) * v[j,c] / l
 *   LSE[i] = m + log(l)                                  (natural log)
 *
 * Subtracting m before exp() is the usual overflow guard; it cancels exactly
 * in O and is added back in LSE.  LSE (the log of the softmax denominator of
 * the scaled, masked scores) is not on the pages; it is the per-row
 * statistic the kernel also returns.
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.
 * Layout: [B, H, N, d] contiguous, d fastest.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* One query row: row index r = (b*H + h)*N + i.  Writes d doubles to o_row
 * and one double to lse_row.  s is caller scratch of at least N doubles. */
static void attn_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int64_t N, int64_t d, int causal, double scale,
                     int64_t r, double *s, double *o_row, double *lse_row) {
  const int64_t bh = r / N;
  const int64_t i = r % N;
  const uint16_t *qi = q + r * d;
  const uint16_t *kb = k + bh * N * d;
  const uint16_t *vb = v + bh * N * d;
  const int64_t nj = causal ? i + 1 : N;

  /* scores of the visible keys */
  double m = -INFINITY;
  for (int64_t j = 0; j < nj; ++j) {
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c)
      acc += bf16_to_double(qi[c]) * bf16_to_double(kb[j * d + c]);
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }

  /* softmax denominator and the weighted sum of V */
  double l = 0.0;
  for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
  for (int64_t j = 0; j < nj; ++j) {
    const double p = exp(s[j] - m);
    l += p;
    for (int64_t c = 0; c < d; ++c) o_row[c] += p * bf16_to_double(vb[j * d + c]);
  }
  for (int64_t c = 0; c < d; ++c) o_row[c] /= l;
  *lse_row = m + log(l);
}

/*
 * attn_ref_f64: q, k, v are host bf16 bits [B,H,N,d].
 *   rows == NULL: every row is computed; o is [B*H*N, d], lse is [B*H*N].
 *   rows != NULL: only the nrows flat row indices listed (each in
 *                 [0, B*H*N)) are computed; o is [nrows, d], lse [nrows].
 *   nthreads <= 0 uses the OpenMP default.
 * Returns 0, or -1 on a bad argument (nothing written).
 */
int attn_ref_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 double *o, double *lse, int64_t B, int64_t H, int64_t N,
                 int64_t d, int causal, double scale, int nthreads,
                 const int64_t *rows, int64_t nrows) {
  if (!q || !k || !v || !o || !lse) return -1;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return -1;
  const int64_t total = B * H * N;
  const int64_t n_out = rows ? nrows : total;
  if (rows) {
    if (nrows < 0) return -1;
    for (int64_t t = 0; t < nrows; ++t)
      if (rows[t] < 0 || rows[t] >= total) return -1;
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    if (!s) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (int64_t t = 0; t < n_out; ++t) {
        const int64_t r = rows ? rows[t] : t;
        attn_row(q, k, v, N, d, causal, scale, r, s, o + t * d, lse + t);
      }
      free(s);
    }
  }
  return failed ? -1 : 0;
}

/*
 * The same definition for queries and keys of different lengths, with K/V
 * heads shared by groups of query heads and a causal offset:
 *
 *   q [B, H, N_q, d],  k and v [B, H_kv, N_k, d];  query head h reads K/V
 *   head h / (H / H_kv) of its batch;
 *   J(i) = {0 .. N_k-1}                   (causal == 0)
 *        = {j < N_k : j <= i + delta}     (causal != 0)
 *
 * A row whose J(i) is empty has no weights to normalise: its result is
 * O = 0 and LSE = log(0) = -inf (the empty sum).  With N_q = N_k, H_kv = H
 * and delta = 0 this is attn_ref_f64.
 */
static void attn_row_general(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             int64_t H, int64_t H_kv, int64_t N_q, int64_t N_k,
                             int64_t d, int causal, int64_t delta, double scale,
                             int64_t r, double *s, double *o_row, double *lse_row) {
  const int64_t bh = r / N_q;
  const int64_t i = r % N_q;
  const int64_t b = bh / H, h = bh % H;
  const int64_t bkv = b * H_kv + h / (H / H_kv);
  const uint16_t *qi = q + r * d;
  const uint16_t *kb = k + bkv * N_k * d;
  const uint16_t *vb = v + bkv * N_k * d;
  int64_t nj = N_k;
  if (causal) {
    const int64_t last = i + delta; /* last visible key */
    nj = last < 0 ? 0 : (last + 1 < N_k ? last + 1 : N_k);
  }
  for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
  if (nj == 0) {
    *lse_row = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int64_t j = 0; j < nj; ++j) {
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c)
      acc += bf16_to_double(qi[c]) * bf16_to_double(kb[j * d + c]);
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int64_t j = 0; j < nj; ++j) {
    const double p = exp(s[j] - m);
    l += p;
    for (int64_t c = 0; c < d; ++c) o_row[c] += p * bf16_to_double(vb[j * d + c]);
  }
  for (int64_t c = 0; c < d; ++c) o_row[c] /= l;
  *lse_row = m + log(l);
}

/*
 * attn_ref_general_f64: q host bf16 bits [B,H,N_q,d]; k, v [B,H_kv,N_k,d].
 *   rows == NULL: every row; o is [B*H*N_q, d], lse [B*H*N_q].
 *   rows != NULL: the nrows flat row indices (b*H + h)*N_q + i listed.
 * Returns 0, or -1 on a bad argument (nothing written).
 */
int attn_ref_general_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         double *o, double *lse, int64_t B, int64_t H, int64_t H_kv,
                         int64_t N_q, int64_t N_k, int64_t d, int causal, int64_t delta,
                         double scale, int nthreads, const int64_t *rows, int64_t nrows) {
  if (!q || !k || !v || !o || !lse) return -1;
  if (B <= 0 || H <= 0 || H_kv <= 0 || H % H_kv != 0 || N_q <= 0 || N_k <= 0 || d <= 0)
    return -1;
  const int64_t total = B * H * N_q;
  const int64_t n_out = rows ? nrows : total;
  if (rows) {
    if (nrows < 0) return -1;
    for (int64_t t = 0; t < nrows; ++t)
      if (rows[t] < 0 || rows[t] >= total) return -1;
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int failed = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N_k);
    if (!s) {
#pragma omp atomic write
      failed = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (int64_t t = 0; t < n_out; ++t) {
        const int64_t r = rows ? rows[t] : t;
        attn_row_general(q, k, v, H, H_kv, N_q, N_k, d, causal, delta, scale, r, s,
                         o + t * d, lse + t);
      }
      free(s);
    }
  }
  return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int attn_ref_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
