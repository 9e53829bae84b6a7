/*
 * kda_ref.h -- the oracle for the Kimi Delta Attention (KDA) core.
 *
 * TEST INFRASTRUCTURE ONLY.  This header and kda_ref.c are the slow,
 * sequential, fp64 statement of what the GPU library computes.  Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load
 * them.  The GPU library shares no code, header or constant with this file.
 *
 * What is computed (per sequence n, per head h, tokens t = 1..T_n in order):
 *
 *   S  <- Diag(exp g_t) S                    channel-wise forget gate on the
 *                                            key rows of the state
 *   u  =  beta_t (v_t - S^T k_t)             delta-rule prediction error
 *   S  <- S + k_t u^T                        rank-1 write; together with the
 *                                            line above this is the generalised
 *                                            Householder transition
 *                                            (I - beta k k^T) Diag(e^g) S + beta k v^T
 *   o_t = scale * S^T q_t                    read-out after the write
 *   if gate != NULL:
 *      o_t <- o_t / sqrt(mean_j o_t[j]^2 + eps) * w * sigmoid(gate_t)
 *
 * Sources: the delta rule built on the generalised Householder transformation
 * ("Kimi K3 from Moonshot AI: 2.8 Trillion Parameters Unveiled", section
 * "Kimi Delta Attention (KDA)"); the per-channel forget gate, fixed-size state
 * and head-wise RMSNorm followed by an input-dependent output gate
 * ("Kimi K3 Architecture Explained", section "Token mixing: what KDA is and
 * why 3:1"); the channel-wise forget gate with log-decay bounded below by
 * g_min = -5 ("Kimi K3: Engineering a 2.8 Trillion Parameter Frontier",
 * section "Dimension 1: Sequence Length via Hybrid KDA-Gated MLA").
 *
 * Layouts (row-major, contiguous):
 *   q, k, g      [T_tot, H, dk]      float (bf16 and fp32 values are exact in float)
 *   v, gate      [T_tot, H, dv]      float
 *   beta         [T_tot, H]          float
 *   norm_weight  [dv]                float or NULL (= all ones)
 *   states       [N, H, dk, dv]      double, row index = key channel
 *   out          [T_tot, H, dv]      double
 *   cu_seqlens   [N + 1]             int64, cu_seqlens[0] = 0, non-decreasing
 */
#ifndef KDA_REF_H
#define KDA_REF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* mode bits */
#define KDA_REF_ERASE_OFF 1u /* test-only: drop the "- S^T k" term: u = beta v (gated linear attention) */
/* pre-processing of the raw projections (see prep_token in kda_ref.c) */
#define KDA_REF_G_LOGITS 2u    /* g holds decay logits a: g = KDA_REF_G_MIN * sigmoid(a) */
#define KDA_REF_BETA_LOGITS 4u /* beta holds logits b: beta = sigmoid(b) */
#define KDA_REF_QK_L2NORM 8u   /* q, k <- x / sqrt(sum x^2 + KDA_REF_L2NORM_EPS) per (token, head) */
#define KDA_REF_G_MIN (-5.0)
#define KDA_REF_L2NORM_EPS 1e-6

/* Return codes */
#define KDA_REF_OK 0
#define KDA_REF_BAD_ARG 1

/* Whole packed batch.  initial_state may be NULL (zeros); final_state may be
 * NULL.  num_threads <= 0 uses the OpenMP default.  Units (sequence, head) run
 * in parallel; tokens inside a unit run in order. */
int kda_ref_forward(int64_t num_seqs, const int64_t* cu_seqlens, int32_t H,
                    int32_t dk, int32_t dv, const float* q, const float* k,
                    const float* v, const float* g, const float* beta,
                    const float* gate, const float* norm_weight,
                    const double* initial_state, double scale, double eps,
                    uint32_t mode, int32_t num_threads, double* out,
                    double* final_state);

/* kda_ref_forward, and also the state after every multiple of snapshot_interval
 * tokens of each sequence: snapshot p of sequence n (p = I, 2I, .., floor(len_n/I) I)
 * is row base_n + p/I - 1 of snapshots [rows, H, dk, dv], base_n = sum_{m<n}
 * floor(len_m / I).  The state S_p is the recurrence's own state after token p. */
int kda_ref_forward_snapshots(int64_t num_seqs, const int64_t* cu_seqlens, int32_t H,
                              int32_t dk, int32_t dv, const float* q, const float* k,
                              const float* v, const float* g, const float* beta,
                              const float* gate, const float* norm_weight,
                              const double* initial_state, double scale, double eps,
                              uint32_t mode, int32_t num_threads, double* out,
                              double* final_state, int64_t snapshot_interval,
                              double* snapshots);

/* One decode step: one new token per sequence.  Inputs are [N, H, d];
 * state is [num_slots, H, dk, dv] updated in place; sequence n uses slot
 * state_indices[n] (or n when state_indices is NULL). */
int kda_ref_decode_step(int64_t N, int32_t H, int32_t dk, int32_t dv,
                        const float* q, const float* k, const float* v,
                        const float* g, const float* beta, const float* gate,
                        const float* norm_weight, double* state,
                        const int64_t* state_indices, double scale, double eps,
                        uint32_t mode, int32_t num_threads, double* out);

/* Number of OpenMP threads a parallel region of the oracle would use. */
int kda_ref_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
