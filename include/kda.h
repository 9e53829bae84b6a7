/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) core library, libkda.so.
 *
 * KDA is a gated delta-rule linear attention with a channel-wise forget gate.
 * Per (sequence, head) it keeps a dk x dv fp32 state S (row = key channel) and,
 * token by token,
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t                      (scale = 1/sqrt(dk) by default)
 *     y_t = o_t / sqrt(mean_j o_t[j]^2 + eps) * w * sigmoid(gate_t)   (when gate != NULL)
 *
 * Sources of each part:
 *   - delta rule on the generalised Householder transformation, chunkwise
 *     ("piecewise parallel") form: "Kimi K3 from Moonshot AI: 2.8 Trillion
 *     Parameters Unveiled", section "Kimi Delta Attention (KDA)";
 *   - fixed-size state, constant per-token decode cost, per-channel forgetting,
 *     head-wise RMSNorm followed by an input-dependent output gate, bounded
 *     log-decay that lets every causal tile be a dense tensor-core product:
 *     "Kimi K3 Architecture Explained: KDA, Attention Residuals and LatentMoE",
 *     section "Token mixing: what KDA is and why 3:1";
 *   - g_min = -5, so a 16-token tile's cumulative log-decay lies in (-80, 0) and
 *     its reciprocal factors (<= e^80) fit the BF16 range: "Kimi K3: Engineering a
 *     2.8 Trillion Parameter Frontier", section "Dimension 1: Sequence Length via
 *     Hybrid KDA-Gated MLA".
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous, 16-byte aligned (beta: aligned to its element size).  Exceptions are
 *     marked HOST.
 *   - The library allocates no memory, never synchronises the stream (except
 *     kda_read_device_error) and launches its kernels on the given cudaStream_t
 *     (passed as void*; NULL = the legacy default stream).
 *   - Host-detectable errors (NULL pointers, shapes, alignment, dtype, workspace
 *     size) return before anything is launched.  A failed launch returns
 *     KDA_ERR_CUDA.  Errors found on the device (a decay outside [g_min, 0] or a
 *     bad state index in checked mode, a bounded wait that ran out) are written to a
 *     device error word and read back with kda_read_device_error.
 *   - Precondition: every g lies in [KDA_G_MIN, 0].  Without KDA_FLAG_CHECK_DECAY a
 *     value below KDA_G_MIN is undefined behaviour for the bf16 tensor-core path
 *     (its tile factors may overflow); with the flag the kernel reports
 *     KDA_ERR_DECAY_OUT_OF_RANGE in the error word.  With KDA_FLAG_G_LOGITS the kernels
 *     compute g = KDA_G_MIN * sigmoid(a) themselves and the bound holds by construction.
 *   - Outputs must not alias inputs.  Decode updates `state` in place by design.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_VERSION_MAJOR 0
#define KDA_VERSION_MINOR 1

/* Lower bound of the per-token log-decay (scaled-sigmoid floor). */
#define KDA_G_MIN (-5.0f)

typedef enum kda_status {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARGUMENT = 1,   /* NULL pointer, bad shape, misaligned pointer, bad cu_seqlens */
  KDA_ERR_UNSUPPORTED = 2,        /* valid request this build does not implement (e.g. dk = 96) */
  KDA_ERR_WORKSPACE_TOO_SMALL = 3,
  KDA_ERR_CUDA = 4,               /* a CUDA runtime call or kernel launch failed */
  KDA_ERR_TIMEOUT = 5,            /* (device) a bounded wait inside a kernel ran out */
  KDA_ERR_DECAY_OUT_OF_RANGE = 6, /* (device, checked mode) some g outside [KDA_G_MIN, 0] */
  KDA_ERR_BAD_STATE_INDEX = 7     /* (device) state_indices[n] outside [0, num_slots): unit skipped */
} kda_status;

typedef enum kda_dtype {
  KDA_BF16 = 0, /* q, k, v, g, beta, gate and out in bfloat16 */
  KDA_F32 = 1   /* the same tensors in float32 */
} kda_dtype;

/* flags (bitwise OR) */
#define KDA_FLAG_CHECK_DECAY 0x1u      /* verify g in [KDA_G_MIN, 0] (and state indices) on the device */
#define KDA_FLAG_FORCE_SIMT 0x2u       /* prefill: use the fp32 CUDA-core chunk kernel even for bf16 */
#define KDA_FLAG_TEST_FORCE_TIMEOUT 0x4u /* tests only: bounded waits give up at once -> KDA_ERR_TIMEOUT */
/* Pre-processing of the raw projections inside the kernels (prefill and decode), so that no
 * separate pass reads and writes q, k, g and beta.  g_min = KDA_G_MIN: the scaled-sigmoid decay
 * bound ("Kimi K3: Engineering a 2.8 Trillion Parameter Frontier", section "Dimension 1"; "Kimi
 * K3 Architecture Explained", section "Token mixing"), which then holds by construction.  The L2
 * norm makes the keys unit vectors, which the delta rule's Householder form assumes ("Kimi K3
 * from Moonshot AI", section "Kimi Delta Attention (KDA)"); the pages do not give its epsilon:
 * x / sqrt(sum x^2 + 1e-6) is taken here. */
#define KDA_FLAG_G_LOGITS 0x8u     /* g holds decay logits a: the kernels use g = KDA_G_MIN * sigmoid(a) */
#define KDA_FLAG_BETA_LOGITS 0x10u /* beta holds logits b: the kernels use sigmoid(b) */
#define KDA_FLAG_QK_L2NORM 0x20u   /* q, k L2-normalised per (token, head): x / sqrt(sum_i x_i^2 + 1e-6) */
#define KDA_L2NORM_EPS 1e-6f
#define KDA_FLAG_DECODE_NO_COMMIT 0x40u /* decode: leave `state` unchanged (verify pass; see tokens) */
/* Unbounded decay: g may be any value <= 0, as with the negative-softplus decay g = -log(1 + e^a)
 * that K3's bounded sigmoid replaced ("Kimi K3 Architecture Explained", section "Token mixing";
 * "Kimi K3 from Moonshot AI", section "Kimi Delta Attention (KDA)").  Prefill then runs on the
 * fp32 CUDA-core kernel with the intra-chunk Gram blocks formed pair by pair (no factor above 1),
 * since the tensor-core tiles rely on the bound; decode handles any g.  With
 * KDA_FLAG_CHECK_DECAY only g > 0 (or NaN) is reported.  The difference in speed between this
 * path and the default one is what the bound buys. */
#define KDA_FLAG_UNBOUNDED_DECAY 0x80u

/* ------------------------------------------------------------------------------------------
 * Chunkwise prefill.
 *
 * Shapes (T_tot = total_tokens, N = num_seqs):
 *   q, k, g       [T_tot, H, dk]   dtype
 *   v, gate       [T_tot, H, dv]   dtype   (gate = gate logits; NULL => no RMSNorm/gate
 *                                            epilogue, out = raw scale * S^T q)
 *   beta          [T_tot, H]       dtype
 *   norm_weight   [dv]             float32 or NULL (= all ones)
 *   initial_state [N, H, dk, dv]   float32 or NULL (= zeros)
 *   out           [T_tot, H, dv]   dtype
 *   final_state   [N, H, dk, dv]   float32 or NULL (not written)
 *   cu_seqlens    HOST int32 [N + 1]: sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]);
 *                 cu_seqlens[0] = 0, non-decreasing, cu_seqlens[N] = T_tot (zero-length
 *                 sequences are allowed: their final state is their initial state).
 *                 NULL => N sequences of T_tot / N tokens each (a dense [N, T, H, d] batch).
 *   dk, dv in {64, 128}.  bf16 with dk = dv = 128 runs the tcgen05 tensor-core kernel;
 *   every other combination (and KDA_FLAG_FORCE_SIMT) runs the fp32 CUDA-core kernel.
 *   split_segments: 0 = automatic; 1 = never split a sequence; P > 1 = split every
 *   sequence into P segments processed in parallel (state carried by a combine pass).
 *   workspace: device scratch of at least kda_chunk_fwd_workspace_size() bytes, 256-byte
 *   aligned, owned by the caller, not shared by calls that may overlap on the GPU.  Its
 *   first 4 bytes are the device error word, cleared at the start of every call.
 * ------------------------------------------------------------------------------------------ */
typedef struct kda_chunk_args {
  int32_t num_seqs;
  int64_t total_tokens;
  const int32_t* cu_seqlens; /* HOST */
  int32_t H, dk, dv;
  kda_dtype dtype;
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  const void* gate;
  const float* norm_weight;
  const float* initial_state;
  void* out;
  float* final_state;
  float scale; /* 0 => 1/sqrt(dk) */
  float eps;   /* RMSNorm epsilon inside the square root (1e-6 in the reference configs) */
  uint32_t flags;
  int32_t split_segments;
  void* workspace;
  size_t workspace_bytes;
  float* snapshots;          /* [n_snap, H, dk, dv] float32 or NULL: chunk-boundary states */
  int32_t snapshot_interval; /* tokens between snapshots: a positive multiple of 64 when
                                snapshots != NULL (ignored otherwise) */
} kda_chunk_args;

/* Chunk-boundary state snapshots (prefix caching: a later call resumes a sequence from the state
 * after any multiple of snapshot_interval tokens, passed as its initial_state).  The pages say that
 * serving reuses earlier work because KDA carries a state instead of a token cache ("What's
 * Actually Inside Kimi K3", section "Vision and Training") and that KDA makes prefix caching a new
 * problem ("What's Kimi K3?", section "The Structure Beneath"); they give no interface.
 *
 * With I = snapshot_interval, sequence n (length len_n) gets snapshots after p = I, 2I, ...,
 * floor(len_n / I) * I tokens: the state S_p of that sequence's recurrence, from its initial state,
 * in the layout of final_state.  Snapshot p of sequence n is row base_n + p / I - 1 of `snapshots`,
 * with base_n = sum over m < n of floor(len_m / I); n_snap = base_N.  A snapshot at p = len_n
 * equals the final state.  The snapshot rows are written by kda_chunk_fwd; nothing else of the
 * buffer is touched.  Errors: snapshots not 16-byte aligned, or I not a positive multiple of 64,
 * -> KDA_ERR_INVALID_ARGUMENT.
 * kda_chunk_fwd_snapshot_count stores n_snap (pure host computation; it reads num_seqs,
 * total_tokens, cu_seqlens and snapshot_interval only, with the same checks as kda_chunk_fwd). */
kda_status kda_chunk_fwd_snapshot_count(const kda_chunk_args* args, int64_t* n_snap);

/* Bytes of workspace kda_chunk_fwd needs for these arguments (pure host computation). */
kda_status kda_chunk_fwd_workspace_size(const kda_chunk_args* args, size_t* bytes);

/* Launch the chunkwise prefill on `cuda_stream`.  Asynchronous. */
kda_status kda_chunk_fwd(const kda_chunk_args* args, void* cuda_stream);

/* ------------------------------------------------------------------------------------------
 * Decode step: K = tokens new tokens (K = 1 by default) for each of N sequences, states
 * updated in place.
 *
 *   q, k, g       [N, K, H, dk]  dtype;  v, gate [N, K, H, dv] dtype (gate NULL => no epilogue)
 *   beta          [N, K, H]      dtype
 *   state         [num_slots, H, dk, dv] float32, read once and (unless
 *                 KDA_FLAG_DECODE_NO_COMMIT) written once, after the K tokens
 *   state_indices [N] int32 device pointer (sequence n uses slot state_indices[n]) or NULL
 *                 (slot n; then num_slots >= N).  Slots used by two sequences race.
 *   out           [N, K, H, dv]  dtype: the output of every position
 *   tokens        K >= 1 (0 is taken as 1): the sequence's next K tokens, in order
 *   position_states [N, K, H, dk, dv] float32 or NULL: the state after each position
 *   error_word    device uint32 or NULL.  Sticky: kernels only set it; the caller zeroes it
 *                 before first use and kda_read_device_error zeroes it after reading.
 *
 * K > 1 serves speculative decoding (the model's multi-token-prediction layer drafts tokens for
 * EAGLE-3 verification: "Kimi K3: Engineering a 2.8 Trillion Parameter Frontier", section
 * "Infrastructure: The Physics of Running a 3T Model"): one call
 * verifies K draft tokens with the state read once.  To roll back to the first m accepted
 * tokens, either keep the position states and take position m - 1 as the new state, or verify
 * with KDA_FLAG_DECODE_NO_COMMIT and then commit with a second call on the m accepted tokens.
 * ------------------------------------------------------------------------------------------ */
typedef struct kda_decode_args {
  int32_t N, H, dk, dv;
  kda_dtype dtype;
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  const void* gate;
  const float* norm_weight;
  float* state;
  int32_t num_slots;
  const int32_t* state_indices;
  void* out;
  float scale; /* 0 => 1/sqrt(dk) */
  float eps;
  uint32_t flags;
  uint32_t* error_word;
  int32_t tokens;
  float* position_states;
} kda_decode_args;

kda_status kda_decode_step(const kda_decode_args* args, void* cuda_stream);

/* ------------------------------------------------------------------------------------------
 * kda_chunk_fwd without a caller-provided workspace.  The paper has no counterpart: this is a
 * deployment convenience for callers that cannot allocate device memory themselves, e.g. code
 * running inside a CUDA graph that is being captured, or inside an inference runtime whose
 * memory pool is fixed at start-up.  Such callers still pass inputs and outputs, but instead of
 * args->workspace (ignored) the call uses a scratch array that the library holds in static
 * device memory: KDA_NOALLOC_SCRATCH_BYTES on every GPU that loads the library, kept until the
 * process exits.
 *   - A request needing more scratch than that (see kda_chunk_fwd_workspace_size; long
 *     sequences split across SMs need the most) returns KDA_ERR_WORKSPACE_TOO_SMALL before
 *     anything is launched.
 *   - The first call on each device looks up the array's device address with that device
 *     current; make that first call before any stream capture.  No call allocates memory.
 *   - All calls share the one array: calls that may overlap on the GPU (different streams,
 *     concurrent threads) race on it.  Serialise them, or use kda_chunk_fwd with a workspace.
 *   - The array keeps the last call's contents; each call clears the error word it needs.
 *   - error_word (may be NULL) receives the device address of the error word for
 *     kda_read_device_error; it stays valid, and is overwritten by the next call.
 * ------------------------------------------------------------------------------------------ */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
kda_status kda_chunk_fwd_noalloc(const kda_chunk_args* args, void* cuda_stream, const void** error_word);

/* Synchronise `cuda_stream`, read the device error word (a kda_chunk_fwd workspace or a
 * decode error_word), reset it to zero and return the status it held (KDA_OK if none).
 * Returns KDA_ERR_CUDA if the synchronisation or the copy fails. */
kda_status kda_read_device_error(const void* error_word, void* cuda_stream);

/* Static, NUL-terminated name of a status code. */
const char* kda_status_string(kda_status status);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H */
