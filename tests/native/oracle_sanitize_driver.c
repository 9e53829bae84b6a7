/*
 * oracle_sanitize_driver.c -- runs the oracle (oracle/kda_ref.c) under AddressSanitizer and
 * UndefinedBehaviorSanitizer: every entry point, every mode bit, ragged and zero-length
 * sequences, snapshots, decode with a slot map, and the argument checks.  Test infrastructure:
 * built and run by tests/test_host_sanitizers.py.  Exits 0 when every call returned what it
 * should and every output is finite; the sanitizers abort on any memory or UB error.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "kda_ref.h"

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static double urand(void) { /* xorshift64*, uniform in [0, 1) */
  rng_state ^= rng_state >> 12;
  rng_state ^= rng_state << 25;
  rng_state ^= rng_state >> 27;
  return (double)((rng_state * 2685821657736338717ull) >> 11) / 9007199254740992.0;
}
static float* fill(size_t n, double lo, double hi) {
  float* p = (float*)malloc(sizeof(float) * (n ? n : 1));
  for (size_t i = 0; i < n; ++i) p[i] = (float)(lo + (hi - lo) * urand());
  return p;
}
static int finite_all(const double* p, size_t n) {
  for (size_t i = 0; i < n; ++i)
    if (!isfinite(p[i])) return 0;
  return 1;
}
#define CHECK(c)                                             \
  do {                                                       \
    if (!(c)) {                                              \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                              \
    }                                                        \
  } while (0)

int main(void) {
  const int32_t H = 2, dk = 8, dv = 5;
  const int64_t cu[] = {0, 0, 1, 18, 58};
  const int64_t N = 4, T = 58;
  float* q = fill((size_t)T * H * dk, -1, 1);
  float* k = fill((size_t)T * H * dk, -1, 1);
  float* v = fill((size_t)T * H * dv, -1, 1);
  float* g = fill((size_t)T * H * dk, -5, 0);
  float* beta = fill((size_t)T * H, 0, 1);
  float* gate = fill((size_t)T * H * dv, -2, 2);
  float* w = fill((size_t)dv, 0.5, 1.5);
  double* s0 = (double*)malloc(sizeof(double) * N * H * dk * dv);
  for (int64_t i = 0; i < N * H * dk * dv; ++i) s0[i] = 0.02 * (urand() - 0.5);
  double* out = (double*)calloc((size_t)T * H * dv, sizeof(double));
  double* fin = (double*)calloc((size_t)N * H * dk * dv, sizeof(double));
  const uint32_t modes[] = {0u, KDA_REF_ERASE_OFF, KDA_REF_G_LOGITS | KDA_REF_BETA_LOGITS | KDA_REF_QK_L2NORM};
  for (int m = 0; m < 3; ++m) {
    CHECK(kda_ref_forward(N, cu, H, dk, dv, q, k, v, g, beta, gate, w, s0, 0.3, 1e-6, modes[m], 1, out,
                          fin) == KDA_REF_OK);
    CHECK(finite_all(out, (size_t)T * H * dv) && finite_all(fin, (size_t)N * H * dk * dv));
    CHECK(kda_ref_forward(N, cu, H, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, modes[m], 1, out,
                          NULL) == KDA_REF_OK);
  }
  /* snapshots every 8 tokens: rows = 0 + 0 + 2 + 5 */
  double* snaps = (double*)calloc((size_t)7 * H * dk * dv, sizeof(double));
  CHECK(kda_ref_forward_snapshots(N, cu, H, dk, dv, q, k, v, g, beta, gate, w, s0, 0.3, 1e-6, 0, 1, out,
                                  fin, 8, snaps) == KDA_REF_OK);
  CHECK(finite_all(snaps, (size_t)7 * H * dk * dv));
  /* decode: 3 sequences into 5 slots through a slot map */
  const int64_t idx[] = {4, 0, 2};
  double* st = (double*)malloc(sizeof(double) * 5 * H * dk * dv);
  for (int64_t i = 0; i < 5 * H * dk * dv; ++i) st[i] = 0.02 * (urand() - 0.5);
  double* dout = (double*)calloc((size_t)3 * H * dv, sizeof(double));
  for (int m = 0; m < 3; ++m) {
    CHECK(kda_ref_decode_step(3, H, dk, dv, q, k, v, g, beta, gate, w, st, idx, 0.3, 1e-6, modes[m], 1, dout) ==
          KDA_REF_OK);
    CHECK(finite_all(dout, (size_t)3 * H * dv) && finite_all(st, (size_t)5 * H * dk * dv));
  }
  CHECK(kda_ref_decode_step(3, H, dk, dv, q, k, v, g, beta, NULL, NULL, st, NULL, 0.3, 1e-6, 0, 1, dout) ==
        KDA_REF_OK);
  /* argument checks */
  const int64_t bad_cu[] = {0, 5, 3};
  CHECK(kda_ref_forward(2, bad_cu, H, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, out, NULL) ==
        KDA_REF_BAD_ARG);
  const int64_t bad_cu0[] = {1, 5};
  CHECK(kda_ref_forward(1, bad_cu0, H, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, out, NULL) ==
        KDA_REF_BAD_ARG);
  CHECK(kda_ref_forward(N, cu, H, dk, dv, NULL, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, out, NULL) ==
        KDA_REF_BAD_ARG);
  CHECK(kda_ref_forward(N, cu, 0, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, out, NULL) ==
        KDA_REF_BAD_ARG);
  CHECK(kda_ref_forward_snapshots(N, cu, H, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, out,
                                  NULL, 0, snaps) == KDA_REF_BAD_ARG);
  CHECK(kda_ref_decode_step(3, H, dk, dv, q, k, v, g, beta, NULL, NULL, NULL, NULL, 0.3, 1e-6, 0, 1, dout) ==
        KDA_REF_BAD_ARG);
  free(q); free(k); free(v); free(g); free(beta); free(gate); free(w); free(s0); free(out); free(fin);
  free(snaps); free(st); free(dout);
  printf("oracle sanitizer driver ok\n");
  return 0;
}
