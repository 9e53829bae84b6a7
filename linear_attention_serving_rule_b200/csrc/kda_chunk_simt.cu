// kda_chunk_simt.cu -- fp32 CUDA-core chunkwise KDA prefill (chunk C = 16).
//
// The chunkwise ("piecewise parallel") form of the recurrence ("Kimi K3 from Moonshot
// AI", section "Kimi Delta Attention (KDA)") for one (segment, head) unit per CTA, all
// in fp32.  With the state S0 at the chunk start and gamma_t the inclusive cumulative
// log-decay from the chunk start (per key channel):
//
//   A_ts = sum_c (k_t e^{gamma_t})_c (k_s e^{-gamma_s})_c   s < t
//   P_ts = sum_c (q_t e^{gamma_t})_c (k_s e^{-gamma_s})_c   s <= t
//   T'   = (I + Diag(beta) A)^-1 Diag(beta)                 forward substitution
//   W    = T' (e^{gamma} k),  U = T' V - W S0
//   O    = scale ((e^{gamma} q) S0 + P U)
//   S    = Diag(e^{gamma_C}) S0 + (e^{gamma_C - gamma} k)^T U
//
// A 16-token chunk keeps |gamma| <= 80 because g >= -5 ("Kimi K3: Engineering a 2.8
// Trillion Parameter Frontier", section "Dimension 1"), so e^{-gamma} <= e^80 is finite in
// fp32 and the chunk-start reference needs no sub-tiling.  This kernel serves the fp32
// workloads and any dk, dv in {64, 128}; it is also the in-library cross-check of the
// tensor-core kernel.
//
// AUG = true runs the split pass 1 on the augmented state [S | M] (dv + dk columns) with
// values augmented by zeros, so M accumulates the segment's transition matrix.
//
// With KDA_FLAG_UNBOUNDED_DECAY the decay may be any g <= 0 (the negative-softplus decay of
// Kimi Linear, which K3 replaced by the bounded sigmoid: "Kimi K3 Architecture Explained",
// section "Token mixing"), so e^{-gamma} may overflow.  A and P are then formed pair by pair
// with e^{gamma_t - gamma_s} <= 1 (s <= t); every other product already uses factors <= 1.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kC = 16;
constexpr int kThreads = 256;

template <int DK, int DV, bool AUG>
struct SimtSmem {
  static constexpr int NS = AUG ? DV + DK : DV;  // state columns
  static constexpr int LDB = DK + 1;              // padded row stride of K e^{-gamma}
  float S[DK * NS];
  float Qt[kC * DK];   // q e^{gamma}
  float Kt[kC * DK];   // k e^{gamma}
  float Kb[kC * LDB];  // k e^{-gamma}
  float Kh[kC * DK];   // k e^{gamma_C - gamma}
  float G[kC * DK];    // gamma
  float V[kC * DV];
  float W[kC * DK];
  float U[kC * NS];
  float O[kC * DV];
  float A[kC * kC];
  float P[kC * kC];
  float Tp[kC * kC];
  float eC[DK];
  float beta[kC];
};

template <typename T, int DK, int DV, bool AUG>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_simt_kernel(const __grid_constant__ Plan plan, const ChunkParams p) {
  using Sm = SimtSmem<DK, DV, AUG>;
  constexpr int NS = Sm::NS;
  constexpr int LDB = Sm::LDB;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm& sm = *reinterpret_cast<Sm*>(smem_raw);

  const int tid = threadIdx.x;
  const int H = plan.H;
  const Seg seg = plan.seg[blockIdx.x / H];
  const int h = blockIdx.x % H;
  const bool checked = (p.flags & KDA_FLAG_CHECK_DECAY) != 0;
  const bool g_logits = (p.flags & KDA_FLAG_G_LOGITS) != 0;
  const bool b_logits = (p.flags & KDA_FLAG_BETA_LOGITS) != 0;
  const bool l2norm = (p.flags & KDA_FLAG_QK_L2NORM) != 0;
  const bool unbounded = (p.flags & KDA_FLAG_UNBOUNDED_DECAY) != 0;
  const bool write_out = (seg.role == kRoleWhole || seg.role == kRoleFromWs);

  // ---- start state
  const float* src = nullptr;
  if (seg.role == kRoleWhole) {
    if (p.initial_state) src = p.initial_state + ((size_t)seg.seq * H + h) * (size_t)(DK * DV);
  } else if (seg.role == kRoleFromWs) {
    src = p.ws_state + ((size_t)seg.slot * H + h) * (size_t)(DK * DV);
  }
  for (int idx = tid; idx < DK * NS; idx += kThreads) {
    const int i = idx / NS, j = idx - (idx / NS) * NS;
    float x;
    if (j < DV) x = src ? src[i * DV + j] : 0.f;
    else x = (j - DV == i) ? 1.f : 0.f;  // M starts as the identity
    sm.S[idx] = x;
  }

  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  const T* g = static_cast<const T*>(p.g);
  const T* bt = static_cast<const T*>(p.beta);
  const T* gate = static_cast<const T*>(p.gate);
  T* out = static_cast<T*>(p.out);

  for (int c0 = 0; c0 < seg.len; c0 += kC) {
    const int L = min(kC, seg.len - c0);
    __syncthreads();  // previous chunk fully consumed
    // ---- load the chunk (rows past the segment end are zero: k = 0, beta = 0, g = 0)
    for (int idx = tid; idx < kC * DK; idx += kThreads) {
      const int t = idx / DK, c = idx - t * DK;
      float qx = 0.f, kx = 0.f, gx = 0.f;
      if (t < L) {
        const size_t r = ((size_t)(seg.tok0 + c0 + t) * H + h) * DK + c;
        qx = to_f32(q[r]); kx = to_f32(k[r]); gx = to_f32(g[r]);
        if (g_logits) gx = KDA_G_MIN / (1.f + expf(-gx));  // g = g_min sigmoid(a)
        if (checked && !((unbounded || gx >= KDA_G_MIN) && gx <= 0.f))
          report_error(p.error_word, KDA_ERR_DECAY_OUT_OF_RANGE);
      }
      sm.Qt[idx] = qx; sm.Kt[idx] = kx; sm.G[idx] = gx;
    }
    for (int idx = tid; idx < kC * DV; idx += kThreads) {
      const int t = idx / DV, j = idx - t * DV;
      sm.V[idx] = (t < L) ? to_f32(v[((size_t)(seg.tok0 + c0 + t) * H + h) * DV + j]) : 0.f;
    }
    if (tid < kC) {
      float b = (tid < L) ? to_f32(bt[(size_t)(seg.tok0 + c0 + tid) * H + h]) : 0.f;
      if (b_logits && tid < L) b = 1.f / (1.f + expf(-b));  // beta = sigmoid(b)
      sm.beta[tid] = b;
    }
    __syncthreads();
    if (l2norm) {  // q, k <- x / sqrt(|x|^2 + eps), one warp per row (padding rows stay zero)
      const int wq = tid >> 5, lq = tid & 31;
      for (int r = wq; r < 2 * kC; r += kThreads / 32) {
        float* xr = (r < kC ? sm.Qt : sm.Kt) + (r % kC) * DK;
        float ss = 0.f;
        for (int c = lq; c < DK; c += 32) ss += xr[c] * xr[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float rn = rsqrtf(ss + KDA_L2NORM_EPS);
        for (int c = lq; c < DK; c += 32) xr[c] *= rn;
      }
      __syncthreads();
    }
    // ---- decay factors: one thread per key channel scans the chunk
    if (tid < DK) {
      const int c = tid;
      float gam = 0.f;
      for (int t = 0; t < kC; ++t) {
        gam += sm.G[t * DK + c];
        sm.G[t * DK + c] = gam;
        const float e = expf(gam);
        const float kx = sm.Kt[t * DK + c];
        // unbounded decay: Kb keeps the raw q for the pairwise Gram blocks
        sm.Kb[t * LDB + c] = unbounded ? sm.Qt[t * DK + c] : kx * expf(-gam);
        sm.Kt[t * DK + c] = kx * e;
        sm.Qt[t * DK + c] *= e;
        sm.Kh[t * DK + c] = kx;  // raw k, scaled below once gamma_C is known
      }
      sm.eC[c] = expf(gam);
      if (!unbounded)
        for (int t = 0; t < kC; ++t) sm.Kh[t * DK + c] *= expf(gam - sm.G[t * DK + c]);
    }
    __syncthreads();
    // ---- decayed Gram blocks A (strict) and P (inclusive): one (t, s) pair per thread
    {
      const int t = tid / kC, s = tid % kC;
      float a = 0.f, pp = 0.f;
      if (!unbounded) {
        for (int c = 0; c < DK; ++c) {
          const float kb = sm.Kb[s * LDB + c];
          a += sm.Kt[t * DK + c] * kb;
          pp += sm.Qt[t * DK + c] * kb;
        }
      } else if (s <= t) {  // raw k (Kh), raw q (Kb) and e^{gamma_t - gamma_s} <= 1
        for (int c = 0; c < DK; ++c) {
          const float f = expf(sm.G[t * DK + c] - sm.G[s * DK + c]);
          const float ks = sm.Kh[s * DK + c];
          a += sm.Kh[t * DK + c] * ks * f;
          pp += sm.Kb[t * LDB + c] * ks * f;
        }
      }
      sm.A[t * kC + s] = (s < t) ? a : 0.f;
      sm.P[t * kC + s] = (s <= t) ? pp : 0.f;
    }
    __syncthreads();
    if (unbounded) {  // now K e^{gamma_C - gamma}
      if (tid < DK) {
        const float gC = sm.G[(kC - 1) * DK + tid];
        for (int t = 0; t < kC; ++t) sm.Kh[t * DK + tid] *= expf(gC - sm.G[t * DK + tid]);
      }
      __syncthreads();
    }
    // ---- T' = (I + Diag(beta) A)^-1 Diag(beta): lane j solves column j
    if (tid < kC) {
      const int j = tid;
      float col[kC];
#pragma unroll
      for (int i = 0; i < kC; ++i) col[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < kC; ++i) {
        if (i > j) {
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < kC; ++m)
            if (m >= j && m < i) acc += sm.A[i * kC + m] * col[m];
          col[i] = -sm.beta[i] * acc;
        }
      }
      const float bj = sm.beta[j];
#pragma unroll
      for (int i = 0; i < kC; ++i) sm.Tp[i * kC + j] = col[i] * bj;
    }
    __syncthreads();
    // ---- W = T' (k e^gamma), U' = T' V (augmented columns of U' are zero)
    for (int idx = tid; idx < kC * DK; idx += kThreads) {
      const int t = idx / DK, c = idx - t * DK;
      float acc = 0.f;
#pragma unroll
      for (int s = 0; s < kC; ++s) acc += sm.Tp[t * kC + s] * sm.Kt[s * DK + c];
      sm.W[idx] = acc;
    }
    for (int idx = tid; idx < kC * NS; idx += kThreads) {
      const int t = idx / NS, j = idx - t * NS;
      float acc = 0.f;
      if (j < DV) {
#pragma unroll
        for (int s = 0; s < kC; ++s) acc += sm.Tp[t * kC + s] * sm.V[s * DV + j];
      }
      sm.U[idx] = acc;
    }
    __syncthreads();
    // ---- U = U' - W S0
    for (int idx = tid; idx < kC * NS; idx += kThreads) {
      const int t = idx / NS, j = idx - t * NS;
      float acc = 0.f;
      for (int i = 0; i < DK; ++i) acc += sm.W[t * DK + i] * sm.S[i * NS + j];
      sm.U[idx] -= acc;
    }
    __syncthreads();
    // ---- O = scale ((q e^gamma) S0 + P U)
    if (write_out) {
      for (int idx = tid; idx < kC * DV; idx += kThreads) {
        const int t = idx / DV, j = idx - t * DV;
        float acc = 0.f;
        for (int i = 0; i < DK; ++i) acc += sm.Qt[t * DK + i] * sm.S[i * NS + j];
        for (int s = 0; s <= t; ++s) acc += sm.P[t * kC + s] * sm.U[s * NS + j];
        sm.O[idx] = p.scale * acc;
      }
    }
    __syncthreads();
    // ---- S = Diag(e^{gamma_C}) S0 + (k e^{gamma_C - gamma})^T U; a chunk that ends on a snapshot
    // boundary also writes S to its snapshot row
    float* snap = nullptr;
    {
      const int e = c0 + L;
      if (seg.snap >= 0 && e >= seg.snap_off && (e - seg.snap_off) % p.snap_interval == 0)
        snap = p.snapshots + ((size_t)(seg.snap + (e - seg.snap_off) / p.snap_interval) * H + h) * (size_t)(DK * DV);
    }
    for (int idx = tid; idx < DK * NS; idx += kThreads) {
      const int i = idx / NS, j = idx - i * NS;
      float acc = sm.eC[i] * sm.S[idx];
#pragma unroll
      for (int t = 0; t < kC; ++t) acc += sm.Kh[t * DK + i] * sm.U[t * NS + j];
      sm.S[idx] = acc;
      if (snap && j < DV) snap[i * DV + j] = acc;
    }
    // ---- epilogue: head-wise RMSNorm * sigmoid(gate), one warp per token
    if (write_out) {
      const int warp = tid >> 5, lane = tid & 31;
      for (int t = warp; t < L; t += kThreads / 32) {
        const size_t r = ((size_t)(seg.tok0 + c0 + t) * H + h) * DV;
        if (gate == nullptr) {
          for (int j = lane; j < DV; j += 32) out[r + j] = from_f32<T>(sm.O[t * DV + j]);
        } else {
          float ss = 0.f;
          for (int j = lane; j < DV; j += 32) { const float o = sm.O[t * DV + j]; ss += o * o; }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          const float rr = rsqrtf(ss / (float)DV + p.eps);
          for (int j = lane; j < DV; j += 32) {
            const float wj = p.norm_weight ? p.norm_weight[j] : 1.f;
            const float sig = 1.f / (1.f + expf(-to_f32(gate[r + j])));
            out[r + j] = from_f32<T>(sm.O[t * DV + j] * rr * wj * sig);
          }
        }
      }
    }
  }
  __syncthreads();
  // ---- end state
  float* dst = nullptr;
  int ld = DV;
  if (seg.role == kRoleWhole || seg.role == kRoleFromWs) {
    if (seg.last && p.final_state) dst = p.final_state + ((size_t)seg.seq * H + h) * (size_t)(DK * DV);
  } else {  // kRoleLocal: [S_loc | M]
    dst = p.ws_local + ((size_t)seg.slot * H + h) * (size_t)(DK * (DV + DK));
    ld = DV + DK;
  }
  if (dst) {
    for (int idx = tid; idx < DK * ld; idx += kThreads) {
      const int i = idx / ld, j = idx - i * ld;
      dst[idx] = sm.S[i * NS + j];
    }
  }
}

template <typename T, int DK, int DV, bool AUG>
cudaError_t launch_t(const Plan& plan, const ChunkParams& p, cudaStream_t stream) {
  const int smem = (int)sizeof(SimtSmem<DK, DV, AUG>);
  auto kern = chunk_simt_kernel<T, DK, DV, AUG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<plan.n_seg * plan.H, kThreads, smem, stream>>>(plan, p);
  return cudaGetLastError();
}

template <typename T, bool AUG>
cudaError_t launch_dims(const Plan& plan, const ChunkParams& p, cudaStream_t stream) {
  if (p.dk == 128 && p.dv == 128) return launch_t<T, 128, 128, AUG>(plan, p, stream);
  if (p.dk == 128 && p.dv == 64) return launch_t<T, 128, 64, AUG>(plan, p, stream);
  if (p.dk == 64 && p.dv == 128) return launch_t<T, 64, 128, AUG>(plan, p, stream);
  return launch_t<T, 64, 64, AUG>(plan, p, stream);
}

}  // namespace

// All segments of one launch share a role class: kRoleLocal launches use the augmented
// state, every other role the plain one.
cudaError_t launch_chunk_simt(const Plan& plan, const ChunkParams& p, kda_dtype dtype, cudaStream_t stream) {
  if (plan.n_seg == 0) return cudaSuccess;
  const bool aug = plan.seg[0].role == kRoleLocal;
  if (dtype == KDA_BF16)
    return aug ? launch_dims<__nv_bfloat16, true>(plan, p, stream) : launch_dims<__nv_bfloat16, false>(plan, p, stream);
  return aug ? launch_dims<float, true>(plan, p, stream) : launch_dims<float, false>(plan, p, stream);
}

}  // namespace kda
