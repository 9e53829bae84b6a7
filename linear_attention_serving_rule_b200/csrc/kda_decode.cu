// kda_decode.cu -- single-token KDA decode step, one CTA per (sequence, head).
//
// The decode step is the recurrence applied to one token with the fixed-size state
// (constant per-token cost: "Kimi K3 Architecture Explained", section "Token mixing"),
// followed by the head-wise RMSNorm and sigmoid output gate of the same section:
//
//   S' = Diag(e^g) S                    channel-wise forget gate on the key rows
//   y_k = S'^T k,  y_q = S'^T q         column reductions over the dk rows
//   u  = beta (v - y_k)                 delta-rule error
//   S  = S' + k u^T                     written back in place
//   o  = scale (y_q + u (k . q))        = scale S^T q after the write
//   out = o / sqrt(mean o^2 + eps) * w * sigmoid(gate)
//
// The step is bound by HBM: the dk x dv fp32 state is read once and written once
// (128 KB per unit at dk = dv = 128); the token's inputs are ~1% of the bytes.  Each
// warp streams one 512-byte state row per 128-bit load, rows are spread over the 8
// warps, and the cross-row reductions go through shared memory.  The state is held in
// registers between the load and the store so it crosses HBM exactly twice.
#include <atomic>

#include "kda_internal.cuh"
#include "ptx_sm100.cuh"

namespace kda {
namespace {

using namespace ptx;

constexpr int kThreads = 256;

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  const void* g;
  const void* beta;
  const void* gate;
  const float* norm_weight;
  float* state;
  const int32_t* state_indices;
  void* out;
  float* position_states;  // [N, K, H, dk, dv] or null
  int32_t H, num_slots, tokens;
  int32_t ahead;  // CTAs resident at once: the unit this many ahead gets its state prefetched
  float scale, eps;
  uint32_t flags;
  uint32_t* error_word;
};

// Two fp32 fused multiply-adds at once (fma.rn.f32x2: each half rounds like fma.rn.f32).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(*reinterpret_cast<const uint64_t*>(&a)),
      "l"(*reinterpret_cast<const uint64_t*>(&b)), "l"(*reinterpret_cast<const uint64_t*>(&c)));
  return *reinterpret_cast<const float2*>(&r);
}
// Two consecutive outputs (4-byte store for bf16, 8-byte for fp32; c is even)
__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }

// Bulk prefetch of [addr, addr + bytes) into L2 (a hint: no completion, no shared memory).
__device__ __forceinline__ void prefetch_l2(const void* addr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(addr), "r"(bytes) : "memory");
}

// kPre: the pre-processing of the raw projections (KDA_FLAG_G_LOGITS, KDA_FLAG_BETA_LOGITS,
// KDA_FLAG_QK_L2NORM) is compiled in; the instance without it is the plain step.
template <typename T, int DK, int DV, bool kPre>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeParams p) {
  constexpr int TPR = DV / 4;              // threads per state row (one float4 each)
  constexpr int RPP = kThreads / TPR;      // rows per pass
  constexpr int NP = DK / RPP;             // passes (float4 registers per thread)
  static_assert(DK % RPP == 0, "rows must divide evenly");

  __shared__ float sk[DK], sq[DK], sa[DK];
  __shared__ __align__(16) float su[DV];
  __shared__ float so[DV];
  __shared__ __align__(16) float red_k[RPP][DV];
  __shared__ __align__(16) float red_q[RPP][DV];
  __shared__ float s_kq, s_rk, s_rq;  // k.q of the normalised vectors; 1/|k|, 1/|q| (or 1)
  __shared__ float s_ss[DV / 32 > 0 ? DV / 32 : 1];

  const int tid = threadIdx.x;
  const int unit = blockIdx.x;
  const int n = unit / p.H;
  const int h = unit - n * p.H;
  const bool checked = (p.flags & KDA_FLAG_CHECK_DECAY) != 0;
  const bool g_logits = kPre && (p.flags & KDA_FLAG_G_LOGITS) != 0;
  const bool l2norm = kPre && (p.flags & KDA_FLAG_QK_L2NORM) != 0;

  int slot = p.state_indices ? p.state_indices[n] : n;
  if (slot < 0 || slot >= p.num_slots) {  // uniform over the block
    if (tid == 0) report_error(p.error_word, KDA_ERR_BAD_STATE_INDEX);
    return;
  }
  float* S = p.state + ((size_t)slot * p.H + h) * (size_t)(DK * DV);

  const int cg = tid % TPR;   // column group: columns 4cg .. 4cg+3
  const int r0 = tid / TPR;   // first row; rows r0 + RPP * i
  float4 s[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i)
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(r0 + RPP * i) * DV) + cg);
  // CTAs start in index order as earlier ones retire, so the unit `ahead` places on is likely to
  // start about when this one ends: pull its state into L2 now, keeping HBM busy across the gap
  // between one CTA's stores and the next one's loads
  if (tid == 0 && p.ahead > 0 && unit + p.ahead < (int)gridDim.x) {
    const int u2 = unit + p.ahead;
    const int n2 = u2 / p.H;
    const int slot2 = p.state_indices ? p.state_indices[n2] : n2;
    if (slot2 >= 0 && slot2 < p.num_slots)
      prefetch_l2(p.state + ((size_t)slot2 * p.H + (u2 - n2 * p.H)) * (size_t)(DK * DV),
                  (uint32_t)(DK * DV * sizeof(float)));
  }

  const int K = p.tokens;
  const bool commit = (p.flags & KDA_FLAG_DECODE_NO_COMMIT) == 0;
  // K tokens of the sequence in order; the state stays in registers between them
  for (int tk = 0; tk < K; ++tk) {
    if (tk > 0) __syncthreads();  // the previous token's shared arrays are consumed
    const size_t row = ((size_t)n * K + tk) * p.H + h;  // token inputs are [N, K, H, d]
    const T* kp = static_cast<const T*>(p.k) + row * DK;
    const T* qp = static_cast<const T*>(p.q) + row * DK;
    const T* gp = static_cast<const T*>(p.g) + row * DK;
    // the token's other inputs are issued now, with k, q and g, and kept in their input type until
    // they are used, so that none of them is a memory round trip of its own later in the step
    T v_raw = T(), gate_raw = T(), beta_raw = T();
    float w_norm = 1.f;
    if (tid < DV) {
      v_raw = static_cast<const T*>(p.v)[row * DV + tid];
      if (p.gate != nullptr) gate_raw = static_cast<const T*>(p.gate)[row * DV + tid];
      if (p.norm_weight) w_norm = p.norm_weight[tid];
    }
    beta_raw = static_cast<const T*>(p.beta)[row];
    for (int i = tid; i < DK; i += kThreads) {
      sk[i] = to_f32(kp[i]);
      sq[i] = to_f32(qp[i]);
      float gi = to_f32(gp[i]);
      if (g_logits) gi = KDA_G_MIN / (1.f + expf(-gi));  // g = g_min sigmoid(a)
      if (checked && !(((p.flags & KDA_FLAG_UNBOUNDED_DECAY) || gi >= KDA_G_MIN) && gi <= 0.0f))
        report_error(p.error_word, KDA_ERR_DECAY_OUT_OF_RANGE);
      sa[i] = expf(gi);
    }
    __syncthreads();
    // With KDA_FLAG_QK_L2NORM the state pass below runs on the raw k and q: S'^T k and S'^T q are
    // linear in them, so 1/|k| and 1/|q| are applied to the reductions and to the write instead.
    if (tid < 32) {
      float acc = 0.f, kk = 0.f, qq = 0.f;
      for (int i = tid; i < DK; i += 32) {
        acc += sk[i] * sq[i];
        if (kPre) {
          kk += sk[i] * sk[i];
          qq += sq[i] * sq[i];
        }
      }
  #pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (kPre) {
          kk += __shfl_xor_sync(0xffffffffu, kk, o);
          qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
      }
      if (tid == 0) {
        const float rk = l2norm ? rsqrtf(kk + KDA_L2NORM_EPS) : 1.f;
        const float rq = l2norm ? rsqrtf(qq + KDA_L2NORM_EPS) : 1.f;
        s_rk = rk;
        s_rq = rq;
        s_kq = acc * rk * rq;
      }
    }

    float4 yk = make_float4(0.f, 0.f, 0.f, 0.f), yq = yk;
  #pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int r = r0 + RPP * i;
      const float a = sa[r], kr = sk[r], qr = sq[r];
      s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
      yk.x += s[i].x * kr; yk.y += s[i].y * kr; yk.z += s[i].z * kr; yk.w += s[i].w * kr;
      yq.x += s[i].x * qr; yq.y += s[i].y * qr; yq.z += s[i].z * qr; yq.w += s[i].w * qr;
    }
    reinterpret_cast<float4*>(red_k[r0])[cg] = yk;
    reinterpret_cast<float4*>(red_q[r0])[cg] = yq;
    __syncthreads();

    float beta = to_f32(beta_raw);
    if (kPre && (p.flags & KDA_FLAG_BETA_LOGITS)) beta = 1.f / (1.f + expf(-beta));  // beta = sigmoid(b)
    const float rk = kPre ? s_rk : 1.f;
    if (tid < DV) {
      float ak = 0.f, aq = 0.f;
  #pragma unroll
      for (int r = 0; r < RPP; ++r) { ak += red_k[r][tid]; aq += red_q[r][tid]; }
      const float u = beta * (to_f32(v_raw) - ak * rk);
      su[tid] = u;
      const float o = p.scale * (kPre ? aq * s_rq + u * s_kq : aq + u * s_kq);
      so[tid] = o;
      if (p.gate != nullptr) {  // the RMSNorm's sum of squares, by warp (read after the next barrier)
        float ss = o * o;
  #pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((tid & 31) == 0) s_ss[tid >> 5] = ss;
      }
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4*>(su)[cg];
  #pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int r = r0 + RPP * i;
      const float kr = sk[r] * rk;
      s[i].x += kr * u4.x; s[i].y += kr * u4.y; s[i].z += kr * u4.z; s[i].w += kr * u4.w;
      if (commit && tk == K - 1) __stcs(reinterpret_cast<float4*>(S + (size_t)r * DV) + cg, s[i]);
    }
    if (p.position_states) {  // the state after this token, for rollback
      float* P = p.position_states + row * (size_t)(DK * DV);
#pragma unroll
      for (int i = 0; i < NP; ++i) __stcs(reinterpret_cast<float4*>(P + (size_t)(r0 + RPP * i) * DV) + cg, s[i]);
    }

    T* op = static_cast<T*>(p.out) + row * DV;
    if (tid < DV) {
      const float o = so[tid];
      if (p.gate == nullptr) {
        op[tid] = from_f32<T>(o);
      } else {  // head-wise RMSNorm over dv (the sums of squares from the solve), then the sigmoid gate
        float tot = 0.f;
  #pragma unroll
        for (int w = 0; w < DV / 32; ++w) tot += s_ss[w];
        const float r = rsqrtf(tot / (float)DV + p.eps);
        const float sig = 1.0f / (1.0f + expf(-to_f32(gate_raw)));
        op[tid] = from_f32<T>(o * r * w_norm * sig);
      }
    }
  }
}

// K > 1 tokens per sequence (speculative verification): the state is read once and written once,
// and the K tokens need only a few block-wide barriers per group of up to KG tokens instead of three
// per token.  With S0 the state before the group, G_j the per-channel cumulative log-decay from the
// group start through token j, and k, q as the recurrence uses them (L2-normalised with
// KDA_FLAG_QK_L2NORM), unrolling the recurrence gives, for j = 1 .. Kg,
//
//   S'_j^T k_j = S0^T (e^{G_j} k_j) + sum_{i<j} u_i c_ji,   c_ji = sum_c k_i[c] k_j[c] e^{G_j[c] - G_i[c]}
//   u_j        = beta_j (v_j - S'_j^T k_j)
//   o_j        = scale (S0^T (e^{G_j} q_j) + sum_{i<=j} u_i d_ji),   d_ji likewise with q_j (d_jj = k_j . q_j)
//   S_j        = Diag(e^{g_j}) S_{j-1} + k_j u_j^T
//
// (S'_j = Diag(e^{g_j}) S_{j-1} is the state the delta rule reads before token j's write).  So one
// pass over the registers forms all 2 Kg column reductions S0^T (e^{G_j} k_j), S0^T (e^{G_j} q_j),
// the small Kg x Kg dots c, d come from the token vectors alone, the u_j and o_j follow column by
// column without further barriers, and the state is then updated token by token in registers (no
// reductions), writing each position's state when asked.  Every input of a group is fetched with
// cp.async before anything waits on it (for the first group, before the state is loaded), so a CTA
// waits for global memory once per group, not once per input.
constexpr int kMultiGroup = 4;  // tokens per group

template <typename T, int DK, int DV>
struct MultiSmem {
  static constexpr int KG = kMultiGroup;
  static constexpr int RPP = kThreads / (DV / 4);
  alignas(16) T rk[KG][DK];  // the group's raw token inputs (cp.async)
  alignas(16) T rq[KG][DK];
  alignas(16) T rg[KG][DK];
  alignas(16) T rv[KG][DV];
  alignas(16) T rgate[KG][DV];
  float sk[KG][DK], sq[KG][DK];   // k, q as loaded (fp32)
  float sg[KG][DK], sa[KG][DK];   // cumulative log-decay G_j from the group start; e^{g_j}
  float skg[KG][DK], sqg[KG][DK]; // k_j e^{G_j}, q_j e^{G_j}
  float ski[KG][DK];              // k_j e^{-G_j} (bounded decay: |G_j| <= 5 KG, so it stays finite)
  float wk[KG][DK];               // e^{G_last - G_j} k_j (normalised): the end state's write factors
  float wK[DK];                   // e^{G_last}: the end state's decay of S0
  alignas(16) float red[RPP][2 * KG][DV];  // column partial sums; then red[0][2 j] = o_j (see below)
  alignas(16) float su[KG][DV];
  float sdot[KG][KG][2];          // [j][i]: raw c_ji (i < j), raw d_ji (i <= j)
  float snrm[KG][2];              // |k_j|^2, |q_j|^2
  float sbeta[KG];
  float sss[KG][DV / 32];         // per warp of the column solve: sum of o_j^2 over its 32 columns
};

template <typename T, int DK, int DV, bool kPre>
__global__ void __launch_bounds__(kThreads, 2) decode_multi_kernel(const DecodeParams p) {
  constexpr int KG = kMultiGroup;
  constexpr int TPR = DV / 4;              // threads per state row (one float4 each)
  constexpr int RPP = kThreads / TPR;      // rows per pass
  constexpr int NP = DK / RPP;             // passes (float4 registers per thread)
  static_assert(DK % RPP == 0, "rows must divide evenly");
  extern __shared__ __align__(16) uint8_t dsm[];
  MultiSmem<T, DK, DV>& sm = *reinterpret_cast<MultiSmem<T, DK, DV>*>(dsm);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int n = unit / p.H;
  const int h = unit - n * p.H;
  const bool checked = (p.flags & KDA_FLAG_CHECK_DECAY) != 0;
  const bool g_logits = kPre && (p.flags & KDA_FLAG_G_LOGITS) != 0;
  const bool l2norm = kPre && (p.flags & KDA_FLAG_QK_L2NORM) != 0;
  const bool b_logits = kPre && (p.flags & KDA_FLAG_BETA_LOGITS) != 0;
  const int K = p.tokens;
  const bool closed = p.position_states == nullptr;  // only the end state is needed

  int slot = p.state_indices ? p.state_indices[n] : n;
  if (slot < 0 || slot >= p.num_slots) {  // uniform over the block
    if (tid == 0) report_error(p.error_word, KDA_ERR_BAD_STATE_INDEX);
    return;
  }
  // the token inputs of the group starting at `base`: 16-byte cp.async chunks, then beta (kept
  // in its input type until the group's inputs are waited for, so that no thread stalls on it
  // before the loads behind it are issued)
  constexpr int CK = DK * (int)sizeof(T) / 16, CV = DV * (int)sizeof(T) / 16;  // chunks per row
  T beta_raw = T();
  auto fetch_group = [&](int base) {
    const int Kg = min(KG, K - base);
    for (int idx = tid; idx < Kg * (3 * CK + 2 * CV); idx += kThreads) {
      const int j = idx / (3 * CK + 2 * CV);
      int c = idx - j * (3 * CK + 2 * CV);
      const size_t row = ((size_t)n * K + base + j) * p.H + h;  // token inputs are [N, K, H, d]
      const T* src;
      uint8_t* dst;
      if (c < 3 * CK) {
        const int t = c / CK;
        c -= t * CK;
        src = static_cast<const T*>(t == 0 ? p.k : t == 1 ? p.q : p.g) + row * DK;
        dst = reinterpret_cast<uint8_t*>(t == 0 ? sm.rk[j] : t == 1 ? sm.rq[j] : sm.rg[j]);
      } else {
        c -= 3 * CK;
        const int t = c / CV;
        c -= t * CV;
        if (t == 1 && p.gate == nullptr) continue;
        src = static_cast<const T*>(t == 0 ? p.v : p.gate) + row * DV;
        dst = reinterpret_cast<uint8_t*>(t == 0 ? sm.rv[j] : sm.rgate[j]);
      }
      cp_async_16(smem_u32(dst + 16 * c), reinterpret_cast<const uint8_t*>(src) + 16 * c);
    }
    cp_async_commit();
    if (tid < Kg) beta_raw = static_cast<const T*>(p.beta)[((size_t)n * K + base + tid) * p.H + h];
  };

  // the state first (the longest wait), then the first group's inputs
  float* S = p.state + ((size_t)slot * p.H + h) * (size_t)(DK * DV);
  const int cg = tid % TPR;   // column group: columns 4cg .. 4cg+3
  const int r0 = tid / TPR;   // first row; rows r0 + RPP * i
  float4 s[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i)
    s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(r0 + RPP * i) * DV) + cg);
  fetch_group(0);
  if (tid == 0 && p.ahead > 0 && unit + p.ahead < (int)gridDim.x) {  // see decode_kernel
    const int u2 = unit + p.ahead;
    const int n2 = u2 / p.H;
    const int slot2 = p.state_indices ? p.state_indices[n2] : n2;
    if (slot2 >= 0 && slot2 < p.num_slots)
      prefetch_l2(p.state + ((size_t)slot2 * p.H + (u2 - n2 * p.H)) * (size_t)(DK * DV),
                  (uint32_t)(DK * DV * sizeof(float)));
  }

  const bool commit = (p.flags & KDA_FLAG_DECODE_NO_COMMIT) == 0;
  for (int base = 0; base < K; base += KG) {
    const int Kg = min(KG, K - base);
    if (base > 0) {
      __syncthreads();  // the previous group's shared arrays are consumed
      fetch_group(base);
    }
    cp_async_wait_all();
    if (tid < Kg) {
      const float beta = to_f32(beta_raw);
      sm.sbeta[tid] = b_logits ? 1.f / (1.f + __expf(-beta)) : beta;  // beta = sigmoid(b)
    }
    __syncthreads();
    // ---- per channel: G_j (prefix over the group), e^{g_j}, and the decayed k, q.  Every thread
    // takes one channel and a run of TPP tokens; it first sums the decay of the tokens before its
    // run, in the same order as the thread of the run before, so G_j is the same value either way.
    {
      constexpr int NPART = kThreads / DK;            // threads per channel
      constexpr int TPP = (KG + NPART - 1) / NPART;   // tokens per thread
      const int c = tid % DK, j0 = (tid / DK) * TPP;
      auto decay = [&](int j) {
        float gi = to_f32(sm.rg[j][c]);
        if (g_logits) gi = KDA_G_MIN / (1.f + __expf(-gi));  // g = g_min sigmoid(a)
        return gi;
      };
      float acc = 0.f;
      for (int j = 0; j < j0 && j < Kg; ++j) acc += decay(j);
      for (int j = j0; j < j0 + TPP && j < Kg; ++j) {
        const float kx = to_f32(sm.rk[j][c]), qx = to_f32(sm.rq[j][c]);
        const float gi = decay(j);
        if (checked && !(((p.flags & KDA_FLAG_UNBOUNDED_DECAY) || gi >= KDA_G_MIN) && gi <= 0.0f))
          report_error(p.error_word, KDA_ERR_DECAY_OUT_OF_RANGE);
        sm.sk[j][c] = kx;
        sm.sq[j][c] = qx;
        if (!closed) sm.sa[j][c] = __expf(gi);  // (only the token-by-token update reads it)
        acc += gi;
        sm.sg[j][c] = acc;
        const float e = __expf(acc);
        sm.skg[j][c] = kx * e;
        sm.sqg[j][c] = qx * e;
        sm.ski[j][c] = kx * __expf(-acc);
      }
    }
    __syncthreads();
    // ---- the token dots and the column reductions over the state.  The 24 dots of a full group
    // (d_ji for i <= j, c_ji for i < j, |k_j|^2, |q_j|^2) are shared out three per warp; each is
    // coded in 6 bits (j, i, kind) and dots of tokens past the group's end are skipped.  With the
    // bounded decay e^{G_j - G_i} = e^{G_j} e^{-G_i} (both finite); with KDA_FLAG_UNBOUNDED_DECAY
    // the factor is formed from the difference, which cannot overflow.
    {
      const bool unbounded = (p.flags & KDA_FLAG_UNBOUNDED_DECAY) != 0;
      // kind 0: c_ji (k_i, k_j), 1: d_ji (k_i, q_j), 2: |k_j|^2, 3: |q_j|^2; code = 16 kind + 4 j + i
      constexpr uint64_t kSlot[3] = {
          // warp w takes 6-bit code w of each word
          (uint64_t)0x10 | (uint64_t)0x15 << 6 | (uint64_t)0x1A << 12 | (uint64_t)0x1F << 18 |
              (uint64_t)0x14 << 24 | (uint64_t)0x18 << 30 | (uint64_t)0x19 << 36 | (uint64_t)0x1C << 42,
          (uint64_t)0x1D << 0 | (uint64_t)0x1E << 6 | (uint64_t)0x04 << 12 | (uint64_t)0x08 << 18 |
              (uint64_t)0x09 << 24 | (uint64_t)0x0C << 30 | (uint64_t)0x0D << 36 | (uint64_t)0x0E << 42,
          (uint64_t)0x20 << 0 | (uint64_t)0x24 << 6 | (uint64_t)0x28 << 12 | (uint64_t)0x2C << 18 |
              (uint64_t)0x30 << 24 | (uint64_t)0x34 << 30 | (uint64_t)0x38 << 36 | (uint64_t)0x3C << 42};
#pragma unroll
      for (int sl = 0; sl < 3; ++sl) {
        const int code = (int)(kSlot[sl] >> (6 * warp)) & 63;
        const int kind = code >> 4, j = (code >> 2) & 3, i = code & 3;
        if (j >= Kg) continue;  // uniform over the warp
        float acc = 0.f;
        if (kind >= 2) {
          const float* x = kind == 3 ? sm.sq[j] : sm.sk[j];
#pragma unroll
          for (int c0 = 0; c0 < DK; c0 += 32) acc += x[c0 + lane] * x[c0 + lane];
        } else {
          const float* xj = kind == 0 ? sm.skg[j] : sm.sqg[j];
          if (!unbounded) {
#pragma unroll
            for (int c0 = 0; c0 < DK; c0 += 32) acc += sm.ski[i][c0 + lane] * xj[c0 + lane];
          } else {
            const float* yj = kind == 0 ? sm.sk[j] : sm.sq[j];
#pragma unroll
            for (int c0 = 0; c0 < DK; c0 += 32) {
              const int c = c0 + lane;
              acc += sm.sk[i][c] * yj[c] * __expf(sm.sg[j][c] - sm.sg[i][c]);
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
          if (kind < 2) sm.sdot[j][i][kind] = acc;
          else sm.snrm[j][kind - 2] = acc;
        }
      }
    }
    // (two tokens per pass over the registers, to keep the accumulators few; column pairs through
    // the two-wide fp32 FMA)
#pragma unroll
    for (int jp = 0; jp < KG; jp += 2) {
      if (jp >= Kg) break;
      float2 acc[4][2];
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m][0] = acc[m][1] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int r = r0 + RPP * i;
        const float2 sl = lo2(s[i]), sh = hi2(s[i]);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = jp + jj;
          if (j < Kg) {
            const float kr = sm.skg[j][r], qr = sm.sqg[j][r];
            const float2 k2 = make_float2(kr, kr), q2 = make_float2(qr, qr);
            acc[2 * jj][0] = ffma2(sl, k2, acc[2 * jj][0]);
            acc[2 * jj][1] = ffma2(sh, k2, acc[2 * jj][1]);
            acc[2 * jj + 1][0] = ffma2(sl, q2, acc[2 * jj + 1][0]);
            acc[2 * jj + 1][1] = ffma2(sh, q2, acc[2 * jj + 1][1]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (2 * jp + m < 2 * Kg)
          reinterpret_cast<float4*>(sm.red[r0][2 * jp + m])[cg] =
              make_float4(acc[m][0].x, acc[m][0].y, acc[m][1].x, acc[m][1].y);
    }
    __syncthreads();
    // ---- column by column: u_j and o_j for the group's tokens in order (o_j goes to red[0][2 j],
    // whose column tid only this thread reads, before it writes it)
    if (tid < DV) {
      float u[KG];
#pragma unroll
      for (int j = 0; j < KG; ++j) {
        if (j >= Kg) break;
        float a = 0.f, bq = 0.f;
#pragma unroll
        for (int r = 0; r < RPP; ++r) { a += sm.red[r][2 * j][tid]; bq += sm.red[r][2 * j + 1][tid]; }
        const float rkj = l2norm ? rsqrtf(sm.snrm[j][0] + KDA_L2NORM_EPS) : 1.f;
        const float rqj = l2norm ? rsqrtf(sm.snrm[j][1] + KDA_L2NORM_EPS) : 1.f;
        float pred = a * rkj, o = bq * rqj;
#pragma unroll
        for (int i = 0; i < KG; ++i) {
          if (i >= j) break;
          const float rki = l2norm ? rsqrtf(sm.snrm[i][0] + KDA_L2NORM_EPS) : 1.f;
          pred += sm.sdot[j][i][0] * rki * rkj * u[i];
          o += sm.sdot[j][i][1] * rqj * rki * u[i];
        }
        u[j] = sm.sbeta[j] * (to_f32(sm.rv[j][tid]) - pred);
        o += sm.sdot[j][j][1] * rqj * rkj * u[j];
        sm.su[j][tid] = u[j];
        const float os = p.scale * o;
        sm.red[0][2 * j][tid] = os;
        if (p.gate != nullptr) {  // the RMSNorm's sum of squares, by warp (read after the next barrier)
          float sq = os * os;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
          if (lane == 0) sm.sss[j][warp] = sq;
        }
      }
    }
    // the end state's factors, on the last DK threads: beside the column solve of the first DV
    static_assert(DK + DV <= kThreads, "the factor threads follow the solve threads");
    if (closed && tid >= kThreads - DK) {
      const int c = tid - (kThreads - DK);
      const float gl = sm.sg[Kg - 1][c];
      sm.wK[c] = __expf(gl);
      for (int j = 0; j < Kg; ++j) {
        const float rkj = l2norm ? rsqrtf(sm.snrm[j][0] + KDA_L2NORM_EPS) : 1.f;
        sm.wk[j][c] = __expf(gl - sm.sg[j][c]) * sm.sk[j][c] * rkj;
      }
    }
    __syncthreads();
    // ---- the state.  With position states: token by token in registers, S_j = Diag(e^{g_j}) S_{j-1}
    // + k_j u_j^T.  Without: the group's end state in one pass, S = Diag(e^{G_last}) S0 +
    // sum_j Diag(e^{G_last - G_j}) k_j u_j^T (the same recurrence unrolled; every factor <= 1).
    if (closed) {
      float2 u2[KG][2];
#pragma unroll
      for (int j = 0; j < KG; ++j) {
        const float4 u4 = j < Kg ? reinterpret_cast<const float4*>(sm.su[j])[cg] : make_float4(0.f, 0.f, 0.f, 0.f);
        u2[j][0] = lo2(u4);
        u2[j][1] = hi2(u4);
      }
      const bool last = base + Kg == K;
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int r = r0 + RPP * i;
        const float dk = sm.wK[r];
        float2 sl = make_float2(s[i].x * dk, s[i].y * dk), sh = make_float2(s[i].z * dk, s[i].w * dk);
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          if (j < Kg) {
            const float w = sm.wk[j][r];
            const float2 w2 = make_float2(w, w);
            sl = ffma2(w2, u2[j][0], sl);
            sh = ffma2(w2, u2[j][1], sh);
          }
        }
        s[i] = make_float4(sl.x, sl.y, sh.x, sh.y);
        if (commit && last) __stcs(reinterpret_cast<float4*>(S + (size_t)r * DV) + cg, s[i]);
      }
    } else {
      for (int j = 0; j < Kg; ++j) {
        const float rkj = l2norm ? rsqrtf(sm.snrm[j][0] + KDA_L2NORM_EPS) : 1.f;
        const float4 u4 = reinterpret_cast<const float4*>(sm.su[j])[cg];
        const bool last = base + j == K - 1;
        const size_t row = ((size_t)n * K + base + j) * p.H + h;
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const int r = r0 + RPP * i;
          const float a = sm.sa[j][r], kr = sm.sk[j][r] * rkj;
          s[i].x = s[i].x * a + kr * u4.x; s[i].y = s[i].y * a + kr * u4.y;
          s[i].z = s[i].z * a + kr * u4.z; s[i].w = s[i].w * a + kr * u4.w;
          if (commit && last) __stcs(reinterpret_cast<float4*>(S + (size_t)r * DV) + cg, s[i]);
        }
        // the state after this token, for rollback
        float* P = p.position_states + row * (size_t)(DK * DV);
#pragma unroll
        for (int i = 0; i < NP; ++i) __stcs(reinterpret_cast<float4*>(P + (size_t)(r0 + RPP * i) * DV) + cg, s[i]);
      }
    }
    // ---- outputs: column pairs of every token of the group over all threads (head-wise RMSNorm
    // over dv from the sums of squares of the solve, then the sigmoid gate)
    for (int idx = tid; idx < Kg * (DV / 2); idx += kThreads) {
      const int j = idx / (DV / 2), c = 2 * (idx - j * (DV / 2));
      const size_t row = ((size_t)n * K + base + j) * p.H + h;
      T* op = static_cast<T*>(p.out) + row * DV + c;
      float y0 = sm.red[0][2 * j][c], y1 = sm.red[0][2 * j][c + 1];
      if (p.gate != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < DV / 32; ++w) ss += sm.sss[j][w];
        const float rr = rsqrtf(ss / (float)DV + p.eps);
        const float w0 = p.norm_weight ? p.norm_weight[c] : 1.0f, w1 = p.norm_weight ? p.norm_weight[c + 1] : 1.0f;
        y0 *= rr * w0 / (1.0f + __expf(-to_f32(sm.rgate[j][c])));
        y1 *= rr * w1 / (1.0f + __expf(-to_f32(sm.rgate[j][c + 1])));
      }
      store2(op, y0, y1);
    }
  }
}

// CTAs of one kernel instance resident on the whole device at once (cached per device; host
// threads that launch at the same time may each compute it and store the same value)
template <typename T, int DK, int DV, bool kPre>
int resident_ctas() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int c = cache[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<T, DK, DV, kPre>, kThreads, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();  // no prefetch then; the launch's own error check must not see this
      return 0;
    }
    c = per_sm * sms > 0 ? per_sm * sms : -1;
    cache[dev].store(c, std::memory_order_relaxed);
  }
  return c > 0 ? c : 0;
}

template <typename T, int DK, int DV, bool kPre>
cudaError_t launch_pre(DecodeParams p, int units, cudaStream_t stream) {
  p.ahead = resident_ctas<T, DK, DV, kPre>();
  if (p.tokens > 1) {
    const int smem = (int)sizeof(MultiSmem<T, DK, DV>);
    auto kern = decode_multi_kernel<T, DK, DV, kPre>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<units, kThreads, smem, stream>>>(p);
  } else
    decode_kernel<T, DK, DV, kPre><<<units, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const DecodeParams& p, int units, cudaStream_t stream) {
  if (p.flags & (KDA_FLAG_G_LOGITS | KDA_FLAG_BETA_LOGITS | KDA_FLAG_QK_L2NORM))
    return launch_pre<T, DK, DV, true>(p, units, stream);
  return launch_pre<T, DK, DV, false>(p, units, stream);
}

template <typename T>
cudaError_t launch_dims(const DecodeParams& p, int dk, int dv, int units, cudaStream_t stream) {
  if (dk == 128 && dv == 128) return launch_t<T, 128, 128>(p, units, stream);
  if (dk == 128 && dv == 64) return launch_t<T, 128, 64>(p, units, stream);
  if (dk == 64 && dv == 128) return launch_t<T, 64, 128>(p, units, stream);
  return launch_t<T, 64, 64>(p, units, stream);
}

}  // namespace

cudaError_t launch_decode(const kda_decode_args& a, cudaStream_t stream) {
  DecodeParams p;
  p.q = a.q; p.k = a.k; p.v = a.v; p.g = a.g; p.beta = a.beta; p.gate = a.gate;
  p.norm_weight = a.norm_weight;
  p.state = a.state;
  p.state_indices = a.state_indices;
  p.out = a.out;
  p.position_states = a.position_states;
  p.tokens = a.tokens > 0 ? a.tokens : 1;
  p.ahead = 0;
  p.H = a.H;
  p.num_slots = a.num_slots;
  p.scale = a.scale;
  p.eps = a.eps;
  p.flags = a.flags;
  p.error_word = a.error_word;
  const int units = a.N * a.H;
  if (units == 0) return cudaSuccess;
  if (a.dtype == KDA_BF16) return launch_dims<__nv_bfloat16>(p, a.dk, a.dv, units, stream);
  return launch_dims<float>(p, a.dk, a.dv, units, stream);
}

}  // namespace kda
