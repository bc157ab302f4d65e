/*
 * Oracle for the k-means assignment step -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/ and bench.py's CPU-baseline leg may load this file's library.
 * The product (the CUDA path) never calls it and shares no code with it.
 *
 * What it computes (page lefilia.fr, Flash-KMeans item): Lloyd's k-means
 * assigns every point to its nearest centroid; the assignment phase
 * compares each of N points with each of K centroids (an N x K distance
 * matrix) and keeps the minimum.  Written out plainly in fp64:
 *
 *   dist[i][j] = sum_c (x[i][c] - cent[j][c])^2
 *   assign[i]  = the smallest j with dist[i][j] = min_j dist[i][j]
 *   best[i]    = min_j dist[i][j]
 *
 * No expansion ||x||^2 - 2 x.c + ||c||^2, no blocking: the differences are
 * squared directly.  Inputs are bf16 bit patterns, widened exactly.
 */
#include <math.h>
#include <stdint.h>
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

/*
 * kmeans_assign_f64: x host bf16 bits [N, d]; cent [K, d].
 *   rows == NULL: every point; assign/best are [N].
 *   rows != NULL: only the nrows listed point indices; assign/best [nrows].
 *   dist (optional, may be NULL): the full [n_out, K] distance rows.
 * Returns 0, or -1 on a bad argument.
 */
int kmeans_assign_f64(const uint16_t *x, const uint16_t *cent, int64_t N, int64_t K, int64_t d,
                      int32_t *assign, double *best, double *dist, const int64_t *rows,
                      int64_t nrows, int nthreads) {
  if (!x || !cent || !assign || !best || N <= 0 || K <= 0 || d <= 0) return -1;
  const int64_t n_out = rows ? nrows : N;
  if (rows) {
    if (nrows < 0) return -1;
    for (int64_t t = 0; t < nrows; ++t)
      if (rows[t] < 0 || rows[t] >= N) return -1;
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < n_out; ++t) {
    const int64_t i = rows ? rows[t] : t;
    double bd = INFINITY;
    int32_t bj = -1;
    for (int64_t j = 0; j < K; ++j) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) {
        const double diff = bf16_to_double(x[i * d + c]) - bf16_to_double(cent[j * d + c]);
        acc += diff * diff;
      }
      if (dist) dist[t * K + j] = acc;
      if (acc < bd) {
        bd = acc;
        bj = (int32_t)j;
      }
    }
    assign[t] = bj;
    best[t] = bd;
  }
  return 0;
}
