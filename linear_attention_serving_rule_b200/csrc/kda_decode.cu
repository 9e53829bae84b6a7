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

namespace kda {
namespace {

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

    float beta = to_f32(static_cast<const T*>(p.beta)[row]);
    if (kPre && (p.flags & KDA_FLAG_BETA_LOGITS)) beta = 1.f / (1.f + expf(-beta));  // beta = sigmoid(b)
    const float rk = kPre ? s_rk : 1.f;
    if (tid < DV) {
      float ak = 0.f, aq = 0.f;
  #pragma unroll
      for (int r = 0; r < RPP; ++r) { ak += red_k[r][tid]; aq += red_q[r][tid]; }
      const float vj = to_f32(static_cast<const T*>(p.v)[row * DV + tid]);
      const float u = beta * (vj - ak * rk);
      su[tid] = u;
      so[tid] = p.scale * (kPre ? aq * s_rq + u * s_kq : aq + u * s_kq);
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
    if (p.gate == nullptr) {
      if (tid < DV) op[tid] = from_f32<T>(so[tid]);
      continue;
    }
    // head-wise RMSNorm over dv, then the sigmoid gate
    float o = 0.f;
    if (tid < DV) {
      o = so[tid];
      float ss = o * o;
  #pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if ((tid & 31) == 0) s_ss[tid >> 5] = ss;
    }
    __syncthreads();
    if (tid < DV) {
      float tot = 0.f;
  #pragma unroll
      for (int w = 0; w < DV / 32; ++w) tot += s_ss[w];
      const float r = rsqrtf(tot / (float)DV + p.eps);
      const float wj = p.norm_weight ? p.norm_weight[tid] : 1.0f;
      const float gl = to_f32(static_cast<const T*>(p.gate)[row * DV + tid]);
      const float sig = 1.0f / (1.0f + expf(-gl));
      op[tid] = from_f32<T>(o * r * wj * sig);
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
