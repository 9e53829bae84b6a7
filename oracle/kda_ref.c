/*
 * kda_ref.c -- the oracle for the Kimi Delta Attention (KDA) core.
 *
 * TEST INFRASTRUCTURE ONLY: the plain, slow, sequential fp64 definition of
 * the recurrence.  Only tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares nothing with the GPU library.  See kda_ref.h for
 * the equations, layouts and the pages each step follows.
 *
 * Every step is written out as the definition states it: no chunking, no
 * reassociation beyond a plain left-to-right sum.  Compiled without
 * -ffast-math so that exp/sqrt and the sums are IEEE double.
 */
#include "kda_ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Head-wise RMSNorm over the dv value channels of one (token, head), then the
 * sigmoid output gate ("Kimi K3 Architecture Explained", section "Token
 * mixing": RMSNorm per head, then an input-dependent gate).  The mean is the
 * biased mean over dv; eps sits inside the square root. */
static void rmsnorm_gate(int32_t dv, double* o, const float* gate,
                         const float* w, double eps) {
  double ss = 0.0;
  for (int32_t j = 0; j < dv; ++j) ss += o[j] * o[j];
  const double r = sqrt(ss / (double)dv + eps);
  for (int32_t j = 0; j < dv; ++j) {
    const double wj = w ? (double)w[j] : 1.0;
    o[j] = o[j] / r * wj * sigmoid((double)gate[j]);
  }
}

/* One token of the gated delta rule on a dk x dv state (row i = key channel i).
 *   1. forget:  S[i][:] *= exp(g[i])
 *   2. error:   u = beta * (v - S^T k)        (erase-off mode: u = beta * v)
 *   3. write:   S += k u^T
 *   4. read:    o = scale * S^T q             (after the write)
 * Steps 1-3 equal S_t = (I - beta k k^T) Diag(e^g) S_{t-1} + beta k v^T. */
static void token_step(int32_t dk, int32_t dv, double* S, const double* q,
                       const double* k, const float* v, const double* g,
                       double beta, double scale, uint32_t mode, double* u,
                       double* o) {
  for (int32_t i = 0; i < dk; ++i) {
    const double a = exp((double)g[i]);
    double* row = S + (size_t)i * dv;
    for (int32_t j = 0; j < dv; ++j) row[j] *= a;
  }
  for (int32_t j = 0; j < dv; ++j) u[j] = 0.0;
  if (!(mode & KDA_REF_ERASE_OFF)) {
    for (int32_t i = 0; i < dk; ++i) {
      const double ki = (double)k[i];
      const double* row = S + (size_t)i * dv;
      for (int32_t j = 0; j < dv; ++j) u[j] += row[j] * ki;
    }
  }
  for (int32_t j = 0; j < dv; ++j) u[j] = beta * ((double)v[j] - u[j]);
  for (int32_t i = 0; i < dk; ++i) {
    const double ki = (double)k[i];
    double* row = S + (size_t)i * dv;
    for (int32_t j = 0; j < dv; ++j) row[j] += ki * u[j];
  }
  for (int32_t j = 0; j < dv; ++j) o[j] = 0.0;
  for (int32_t i = 0; i < dk; ++i) {
    const double qi = (double)q[i];
    const double* row = S + (size_t)i * dv;
    for (int32_t j = 0; j < dv; ++j) o[j] += row[j] * qi;
  }
  for (int32_t j = 0; j < dv; ++j) o[j] *= scale;
}

/* The token's q, k, g and beta as the recurrence uses them, in double.  With the
 * pre-processing mode bits the inputs are the raw projections instead:
 *   KDA_REF_G_LOGITS:    g = g_min * sigmoid(a), g_min = -5 (the scaled-sigmoid
 *                        decay: "Kimi K3: Engineering a 2.8 Trillion Parameter
 *                        Frontier", section "Dimension 1"; "Kimi K3 Architecture
 *                        Explained", section "Token mixing")
 *   KDA_REF_BETA_LOGITS: beta = sigmoid(b)
 *   KDA_REF_QK_L2NORM:   q <- q / sqrt(sum_i q_i^2 + 1e-6), the same for k
 *                        (unit-norm keys are what makes the delta write a
 *                        Householder projection: "Kimi K3 from Moonshot AI",
 *                        section "Kimi Delta Attention (KDA)") */
static double prep_token(int32_t dk, const float* q, const float* k, const float* g,
                         float beta, uint32_t mode, double* qd, double* kd, double* gd) {
  for (int32_t i = 0; i < dk; ++i) {
    qd[i] = (double)q[i];
    kd[i] = (double)k[i];
    gd[i] = (mode & KDA_REF_G_LOGITS) ? KDA_REF_G_MIN * sigmoid((double)g[i]) : (double)g[i];
  }
  if (mode & KDA_REF_QK_L2NORM) {
    double sq = 0.0, sk = 0.0;
    for (int32_t i = 0; i < dk; ++i) {
      sq += qd[i] * qd[i];
      sk += kd[i] * kd[i];
    }
    const double rq = 1.0 / sqrt(sq + KDA_REF_L2NORM_EPS), rk = 1.0 / sqrt(sk + KDA_REF_L2NORM_EPS);
    for (int32_t i = 0; i < dk; ++i) {
      qd[i] *= rq;
      kd[i] *= rk;
    }
  }
  return (mode & KDA_REF_BETA_LOGITS) ? sigmoid((double)beta) : (double)beta;
}

static int check_common(int32_t H, int32_t dk, int32_t dv, const float* q,
                        const float* k, const float* v, const float* g,
                        const float* beta) {
  if (H <= 0 || dk <= 0 || dv <= 0) return KDA_REF_BAD_ARG;
  if (!q || !k || !v || !g || !beta) return KDA_REF_BAD_ARG;
  return KDA_REF_OK;
}

/* The sequential recurrence over every (sequence, head) unit; with snapshots != NULL the state
 * after each multiple of snapshot_interval tokens of a sequence is also copied out (the state
 * S_p of the definition, nothing else). */
static int forward_impl(int64_t num_seqs, const int64_t* cu_seqlens, int32_t H,
                        int32_t dk, int32_t dv, const float* q, const float* k,
                        const float* v, const float* g, const float* beta,
                        const float* gate, const float* norm_weight,
                        const double* initial_state, double scale, double eps,
                        uint32_t mode, int32_t num_threads, double* out,
                        double* final_state, int64_t snapshot_interval,
                        double* snapshots) {
  if (num_seqs < 0 || !cu_seqlens || !out) return KDA_REF_BAD_ARG;
  if (snapshots && snapshot_interval <= 0) return KDA_REF_BAD_ARG;
  if (check_common(H, dk, dv, q, k, v, g, beta)) return KDA_REF_BAD_ARG;
  if (cu_seqlens[0] != 0) return KDA_REF_BAD_ARG;
  for (int64_t n = 0; n < num_seqs; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return KDA_REF_BAD_ARG;

  const int64_t units = num_seqs * (int64_t)H;
  const size_t state_elems = (size_t)dk * (size_t)dv;
  int bad = 0;
  /* snapshot row of sequence n's first snapshot: sum over m < n of floor(len_m / interval) */
  int64_t* snap_base = NULL;
  if (snapshots) {
    snap_base = (int64_t*)malloc(sizeof(int64_t) * (size_t)(num_seqs + 1));
    if (!snap_base) return KDA_REF_BAD_ARG;
    snap_base[0] = 0;
    for (int64_t n = 0; n < num_seqs; ++n)
      snap_base[n + 1] = snap_base[n] + (cu_seqlens[n + 1] - cu_seqlens[n]) / snapshot_interval;
  }
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#else
  (void)num_threads;
#endif

#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * state_elems);
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    double* qkg = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
    if (!S || !u || !qkg) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t unit = 0; unit < units; ++unit) {
      if (!S || !u || !qkg) continue;
      const int64_t n = unit / H;
      const int32_t h = (int32_t)(unit % H);
      if (initial_state)
        memcpy(S, initial_state + (size_t)unit * state_elems,
               sizeof(double) * state_elems);
      else
        memset(S, 0, sizeof(double) * state_elems);
      for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
        const size_t row = (size_t)t * H + h;
        double* o = out + row * dv;
        const double b = prep_token(dk, q + row * dk, k + row * dk, g + row * dk, beta[row],
                                    mode, qkg, qkg + dk, qkg + 2 * dk);
        token_step(dk, dv, S, qkg, qkg + dk, v + row * dv, qkg + 2 * dk, b, scale, mode, u, o);
        if (gate) rmsnorm_gate(dv, o, gate + row * dv, norm_weight, eps);
        const int64_t done = t - cu_seqlens[n] + 1; /* tokens of the sequence consumed */
        if (snapshots && done % snapshot_interval == 0) {
          const int64_t srow = snap_base[n] + done / snapshot_interval - 1;
          memcpy(snapshots + ((size_t)srow * H + h) * state_elems, S,
                 sizeof(double) * state_elems);
        }
      }
      if (final_state)
        memcpy(final_state + (size_t)unit * state_elems, S,
               sizeof(double) * state_elems);
    }
    free(S);
    free(u);
    free(qkg);
  }
  free(snap_base);
  return bad ? KDA_REF_BAD_ARG : KDA_REF_OK;
}

int kda_ref_forward(int64_t num_seqs, const int64_t* cu_seqlens, int32_t H,
                    int32_t dk, int32_t dv, const float* q, const float* k,
                    const float* v, const float* g, const float* beta,
                    const float* gate, const float* norm_weight,
                    const double* initial_state, double scale, double eps,
                    uint32_t mode, int32_t num_threads, double* out,
                    double* final_state) {
  return forward_impl(num_seqs, cu_seqlens, H, dk, dv, q, k, v, g, beta, gate,
                      norm_weight, initial_state, scale, eps, mode, num_threads,
                      out, final_state, 0, NULL);
}

int kda_ref_forward_snapshots(int64_t num_seqs, const int64_t* cu_seqlens, int32_t H,
                              int32_t dk, int32_t dv, const float* q, const float* k,
                              const float* v, const float* g, const float* beta,
                              const float* gate, const float* norm_weight,
                              const double* initial_state, double scale, double eps,
                              uint32_t mode, int32_t num_threads, double* out,
                              double* final_state, int64_t snapshot_interval,
                              double* snapshots) {
  if (!snapshots) return KDA_REF_BAD_ARG;
  return forward_impl(num_seqs, cu_seqlens, H, dk, dv, q, k, v, g, beta, gate,
                      norm_weight, initial_state, scale, eps, mode, num_threads,
                      out, final_state, snapshot_interval, snapshots);
}

int kda_ref_decode_step(int64_t N, int32_t H, int32_t dk, int32_t dv,
                        const float* q, const float* k, const float* v,
                        const float* g, const float* beta, const float* gate,
                        const float* norm_weight, double* state,
                        const int64_t* state_indices, double scale, double eps,
                        uint32_t mode, int32_t num_threads, double* out) {
  if (N < 0 || !state || !out) return KDA_REF_BAD_ARG;
  if (check_common(H, dk, dv, q, k, v, g, beta)) return KDA_REF_BAD_ARG;
  const size_t state_elems = (size_t)dk * (size_t)dv;
  int bad = 0;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#else
  (void)num_threads;
#endif
#pragma omp parallel
  {
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    double* qkg = (double*)malloc(sizeof(double) * 3 * (size_t)dk);
    if (!u || !qkg) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(static)
    for (int64_t unit = 0; unit < N * (int64_t)H; ++unit) {
      if (!u || !qkg) continue;
      const int64_t n = unit / H;
      const int32_t h = (int32_t)(unit % H);
      const int64_t slot = state_indices ? state_indices[n] : n;
      double* S = state + ((size_t)slot * H + h) * state_elems;
      const size_t row = (size_t)unit; /* [N, H] row of the token inputs */
      double* o = out + row * dv;
      const double b = prep_token(dk, q + row * dk, k + row * dk, g + row * dk, beta[row],
                                  mode, qkg, qkg + dk, qkg + 2 * dk);
      token_step(dk, dv, S, qkg, qkg + dk, v + row * dv, qkg + 2 * dk, b, scale, mode, u, o);
      if (gate) rmsnorm_gate(dv, o, gate + row * dv, norm_weight, eps);
    }
    free(u);
    free(qkg);
  }
  return bad ? KDA_REF_BAD_ARG : KDA_REF_OK;
}

int kda_ref_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
