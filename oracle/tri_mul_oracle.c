/*
 * fp64 CPU oracle for the triangle multiplicative update contraction.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file; only the tests and the benchmark's CPU legs do. It shares no code,
 * header or constant with the CUDA library.
 *
 * What it computes. The pages name triangle multiplication beside triangle
 * attention as the second operation of the pair stack that their kernels
 * accelerate ("TurboPairFormer accelera fino a 1,73x l'addestramento di
 * OpenFold3 nei test", sections "Dove si impiega il tempo" and "Benchmark di
 * addestramento") but print no formula. This file takes the standard
 * AlphaFold-family contraction at its core, per channel c, for the two edge
 * directions of a pair (i, j):
 *
 *   outgoing edges: t[c][i][j] = sum_k a[c][i][k] * b[c][j][k]
 *   incoming edges: t[c][i][j] = sum_k a[c][k][i] * b[c][k][j]
 *
 * Tensors are channel-major, x[c][r][s] at (c*N + r)*N + s. The backward of
 * L = sum(dt * t), from the chain rule (t is bilinear in a and b):
 *
 *   outgoing: da[c][i][k] = sum_j dt[c][i][j] b[c][j][k]
 *             db[c][j][k] = sum_i dt[c][i][j] a[c][i][k]
 *   incoming: da[c][k][i] = sum_j dt[c][i][j] b[c][k][j]
 *             db[c][k][j] = sum_i dt[c][i][j] a[c][k][i]
 *
 * Plain loops in the order the sums are written, fp64 accumulation, OpenMP over
 * channels. Inputs are float32 values (the bf16 values the GPU receives, widened
 * without change).
 */
#include <stdint.h>

enum { OUTGOING = 0, INCOMING = 1 };

static int check(int64_t N, int C, int dir) {
  if (N < 0 || C < 1) return 1;
  if (dir != OUTGOING && dir != INCOMING) return 2;
  return 0;
}

/* x[c][r][s] of a channel-major N x N stack */
static double at(const float *x, int64_t N, int c, int64_t r, int64_t s) {
  return (double)x[((int64_t)c * N + r) * N + s];
}

int tri_mul_oracle_fwd(int64_t N, int C, int dir, const float *a, const float *b, double *t) {
  const int rc = check(N, C, dir);
  if (rc) return rc;
#pragma omp parallel for schedule(static)
  for (int c = 0; c < C; ++c)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) {
        double s = 0.0;
        for (int64_t k = 0; k < N; ++k)
          s += dir == OUTGOING ? at(a, N, c, i, k) * at(b, N, c, j, k)
                               : at(a, N, c, k, i) * at(b, N, c, k, j);
        t[((int64_t)c * N + i) * N + j] = s;
      }
  return 0;
}

int tri_mul_oracle_bwd(int64_t N, int C, int dir, const float *a, const float *b,
                       const float *dt, double *da, double *db) {
  const int rc = check(N, C, dir);
  if (rc) return rc;
#pragma omp parallel for schedule(static)
  for (int c = 0; c < C; ++c)
    for (int64_t r = 0; r < N; ++r)
      for (int64_t s = 0; s < N; ++s) {
        double ga = 0.0, gb = 0.0;
        if (dir == OUTGOING) {
          /* da[c][i=r][k=s], db[c][j=r][k=s] */
          for (int64_t j = 0; j < N; ++j) ga += at(dt, N, c, r, j) * at(b, N, c, j, s);
          for (int64_t i = 0; i < N; ++i) gb += at(dt, N, c, i, r) * at(a, N, c, i, s);
        } else {
          /* da[c][k=r][i=s], db[c][k=r][j=s] */
          for (int64_t j = 0; j < N; ++j) ga += at(dt, N, c, s, j) * at(b, N, c, r, j);
          for (int64_t i = 0; i < N; ++i) gb += at(dt, N, c, i, s) * at(a, N, c, r, i);
        }
        da[((int64_t)c * N + r) * N + s] = ga;
        db[((int64_t)c * N + r) * N + s] = gb;
      }
  return 0;
}
