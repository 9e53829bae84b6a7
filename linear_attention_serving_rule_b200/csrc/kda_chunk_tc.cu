// kda_chunk_tc.cu -- tcgen05 tensor-core chunkwise KDA prefill (bf16 in, fp32 accumulate,
// dk = dv = 128, chunk C = 64 = four 16-token sub-tiles).
//
// The chunkwise ("piecewise parallel") form ("Kimi K3 from Moonshot AI", section "Kimi
// Delta Attention (KDA)") for one (segment, head) unit per CTA.  With the state S0 at the
// chunk start and gamma_t the inclusive cumulative log-decay from the chunk start:
//
//   A_ts = sum_c k_t[c] k_s[c] e^{gamma_t[c]-gamma_s[c]} (s < t),  P_ts likewise with q_t (s <= t)
//   T'   = (I + Diag(beta) A)^-1 Diag(beta)
//   W    = T' (e^{gamma} k),   U = T' V - W S0
//   O    = scale ((e^{gamma} q) S0 + P U)          -> RMSNorm * sigmoid(gate) epilogue
//   S    = Diag(e^{gamma_C}) S0 + (e^{gamma_C - gamma} k)^T U
//
// Every product above is a dense tcgen05 UMMA (bf16 x bf16 -> fp32 in TMEM).  The decayed
// Gram blocks A and P are dense too: the log-decay floor g >= -5 keeps the cumulative decay
// of a 16-token sub-tile in (-80, 0), so with the reference point at the start of each row's
// sub-tile both factors of e^{gamma_t - gamma_s} fit bf16 (row factor <= 1, column factor
// <= e^80) -- "Kimi K3: Engineering a 2.8 Trillion Parameter Frontier", section "Dimension 1",
// and "Kimi K3 Architecture Explained", section "Token mixing" (every causal tile a dense
// tensor-core product instead of a per-position loop).  Rows of sub-tile a use column
// operand Kc_a = k e^{r_a - gamma} over the first 16(a+1) tokens; one M=128 UMMA per a
// produces A (rows 0-63) and P (rows 64-127) from the stacked operand [k; q] e^{gamma - r_own}.
//
// Work split (160 threads): warp 4 is the TMA producer (q, k, g | v | gate tiles, released per
// group as soon as the chunk no longer needs them); warps 0-3 are the compute warpgroup:
// thread i owns TMEM lane i and row i of the fp32 state S (kept in registers), builds the
// decayed bf16 operands, the UT inverse T', and runs the epilogue; thread 0 issues the UMMAs.
//
// TMEM (512 columns allocated): [0,128) K^T U (M=128); [128,288) A|P (M=128, N = 16,32,48,64);
// [288,416) W / O at lane offset 0 and U' -> U at lane offset 16 (two interleaved M=64 tiles).
//
// Every wait is bounded (%globaltimer): on expiry the kernel records KDA_ERR_TIMEOUT, stops
// issuing work, drains its own in-flight TMA and UMMA operations (bounded again), frees TMEM
// and returns.
#include <cuda.h>

#include "kda_internal.cuh"
#include "ptx_sm100.cuh"

namespace kda {
namespace {

using namespace ptx;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int kCompute = 128;
constexpr int kThreads = 160;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0, OFF_K = 16384, OFF_G = 32768, OFF_V = 49152, OFF_GATE = 65536;
constexpr uint32_t OFF_S = 81920;    // bf16 state, MN-major [dk rows][dv], two 16 KB column blocks
constexpr uint32_t OFF_R = 114688;   // 72 KB region reused across the phases of a chunk
// phase A (decayed Gram operands)
constexpr uint32_t R_KQ = 0;                                        // [k; q] e^{gamma - r_own}, 128 rows
// Kc_a (16(a+1) rows) at 32768, 36864, 45056, 57344
__host__ __device__ constexpr uint32_t r_kc(int a) { return a == 0 ? 32768u : a == 1 ? 36864u : a == 2 ? 45056u : 57344u; }
// phase B (inverse) and later
constexpr uint32_t R_AF = 0, R_TF = 16640;                          // fp32 [64][65]
constexpr uint32_t R_KT = 0, R_QT = 16384, R_KH = 32768;            // e^g k, e^g q, e^{gC-g} k
constexpr uint32_t R_W = 0, R_U = 0;                                // -W, then U (bf16)
constexpr uint32_t R_TP = 49152, R_P = 57344, R_Y = 65536;          // T', P (bf16), scratch
constexpr uint32_t OFF_MISC = OFF_R + 73728;                        // 188416
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096 + 1024;             // + misc + alignment slack
constexpr int LDF = 65;                                             // fp32 row stride of A, T

constexpr uint32_t TM_KU = 0, TM_AP = 128, TM_WU = 288;
// column offset of the A|P accumulator of sub-tile a (N = 16, 32, 48, 64)
__host__ __device__ constexpr uint32_t ap_off(int a) { return a == 0 ? 0u : a == 1 ? 16u : a == 2 ? 48u : 96u; }

struct Misc {
  uint64_t full_qkg, full_v, full_gate, empty_qkg, empty_v, empty_gate, mma;
  uint32_t tmem_base;
  int32_t abort;
  float beta[C];
  float2 tot[64];
  float ref[5][DK];   // r_0..r_3 and gamma_C per channel (log2 units)
  float ec[DK];       // e^{gamma_C}
};
static_assert(sizeof(Misc) <= 4096, "misc block too large");

struct TcMaps {
  CUtensorMap q, k, g, v, gate;
};

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait by one thread.  Returns false (and sets abort) on expiry or if another thread
// already aborted.  limit_ns = 0 means: give up unless the phase has already completed.
__device__ bool wait_bounded(uint64_t* bar, uint32_t parity, Misc* m, uint64_t limit_ns, uint32_t* err,
                             bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *(volatile int32_t*)&m->abort) return false;
    if ((it & 63u) == 0 && globaltimer() - t0 > limit_ns) {
      *(volatile int32_t*)&m->abort = 1;
      report_error(err, KDA_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void st_u32(uint8_t* base, uint32_t off, uint32_t v) {
  *reinterpret_cast<uint32_t*>(base + off) = v;
}
__device__ __forceinline__ uint32_t ld_u32(const uint8_t* base, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(base + off);
}

// Issue the K loop of one UMMA: A and B descriptors advance by (a_step, b_step) bytes per
// 16-wide K step; K-major 128-wide operands jump to their second 64-column block after 4 steps.
__device__ __forceinline__ void umma_k_loop(uint32_t d, uint32_t a_addr, uint32_t a_lbo, bool a_kmajor,
                                            uint32_t a_blk, uint32_t b_addr, uint32_t b_lbo, bool b_kmajor,
                                            uint32_t b_blk, int ksteps, uint32_t idesc, bool accumulate) {
  for (int k = 0; k < ksteps; ++k) {
    const uint32_t ao = a_kmajor ? (uint32_t)(k >> 2) * a_blk + (uint32_t)(k & 3) * 32u : (uint32_t)k * 2048u;
    const uint32_t bo = b_kmajor ? (uint32_t)(k >> 2) * b_blk + (uint32_t)(k & 3) * 32u : (uint32_t)k * 2048u;
    umma_bf16(d, smem_desc_sw128(a_addr + ao, a_lbo, 1024), smem_desc_sw128(b_addr + bo, b_lbo, 1024), idesc,
              (accumulate || k > 0) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ Plan plan, const __grid_constant__ TcMaps maps, const ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* m = reinterpret_cast<Misc*>(sm + OFF_MISC);
  uint8_t* R = sm + OFF_R;
  const uint32_t sm_u = smem_u32(sm);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = plan.H;
  const Seg seg = plan.seg[blockIdx.x / H];
  const int h = blockIdx.x % H;
  const bool has_gate = p.gate != nullptr;
  const bool checked = (p.flags & KDA_FLAG_CHECK_DECAY) != 0;
  const uint64_t limit = (p.flags & KDA_FLAG_TEST_FORCE_TIMEOUT) ? 0ull : 2000000000ull;  // 2 s
  const uint64_t drain_limit = 2000000000ull;
  const int nchunks = (seg.len + C - 1) / C;

  if (tid == 0) {
    mbar_init(&m->full_qkg, 1); mbar_init(&m->full_v, 1); mbar_init(&m->full_gate, 1);
    mbar_init(&m->empty_qkg, 1); mbar_init(&m->empty_v, 1); mbar_init(&m->empty_gate, 1);
    mbar_init(&m->mma, 1);
    m->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&m->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.g); prefetch_tmap(&maps.v);
    if (has_gate) prefetch_tmap(&maps.gate);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = m->tmem_base;

  if (warp == 4) {
    // ===================================================================== TMA producer
    if (lane == 0) {
      int iq = -1, iv = -1, ig = -1;  // last chunk whose q/k/g, v, gate loads were issued
      for (int j = 0; j < nchunks; ++j) {
        const int32_t tok = seg.tok0 + j * C;
        const uint32_t par = (uint32_t)((j & 1) ^ 1);
        if (!wait_bounded(&m->empty_qkg, par, m, drain_limit, p.error_word)) break;
        mbar_arrive_expect_tx(&m->full_qkg, 3 * 16384);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_3d(sm + OFF_Q + hf * 8192, &maps.q, &m->full_qkg, hf * 64, h, tok);
          tma_load_3d(sm + OFF_K + hf * 8192, &maps.k, &m->full_qkg, hf * 64, h, tok);
          tma_load_3d(sm + OFF_G + hf * 8192, &maps.g, &m->full_qkg, hf * 64, h, tok);
        }
        iq = j;
        if (!wait_bounded(&m->empty_v, par, m, drain_limit, p.error_word)) break;
        mbar_arrive_expect_tx(&m->full_v, 16384);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + OFF_V + hf * 8192, &maps.v, &m->full_v, hf * 64, h, tok);
        iv = j;
        if (has_gate) {
          if (!wait_bounded(&m->empty_gate, par, m, drain_limit, p.error_word)) break;
          mbar_arrive_expect_tx(&m->full_gate, 16384);
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sm + OFF_GATE + hf * 8192, &maps.gate, &m->full_gate, hf * 64, h, tok);
          ig = j;
        }
      }
      // drain: after an abort, wait (bounded, regardless of the abort) for the loads issued
      if (*(volatile int32_t*)&m->abort) {
        if (iq >= 0) wait_bounded(&m->full_qkg, (uint32_t)(iq & 1), m, drain_limit, p.error_word, false);
        if (iv >= 0) wait_bounded(&m->full_v, (uint32_t)(iv & 1), m, drain_limit, p.error_word, false);
        if (ig >= 0) wait_bounded(&m->full_gate, (uint32_t)(ig & 1), m, drain_limit, p.error_word, false);
      }
    }
  } else {
    // ===================================================================== compute warpgroup
    float S[DV];  // row `tid` of the fp32 state
    const size_t unit_state = (size_t)DK * DV;
    {
      const float* src = nullptr;
      if (seg.role == kRoleWhole || seg.role == kRoleHead) {
        if (p.initial_state) src = p.initial_state + ((size_t)seg.seq * H + h) * unit_state;
      } else if (seg.role == kRoleFromWs) {
        src = p.ws_state + ((size_t)seg.slot * H + h) * unit_state;
      }
#pragma unroll
      for (int c = 0; c < DV; c += 4) {
        float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)tid * DV + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[c] = x.x; S[c + 1] = x.y; S[c + 2] = x.z; S[c + 3] = x.w;
      }
#pragma unroll
      for (int c = 0; c < DV; c += 2) st_u32(sm, OFF_S + sw128_off(tid, c, 16384), f2_to_bf2(S[c], S[c + 1]));
    }
    const bool write_out = (seg.role == kRoleWhole || seg.role == kRoleFromWs);
    const int pr = tid & 63, hh = tid >> 6;  // channel pair (2pr, 2pr+1) and token half for the scans
    const int c0 = 2 * pr;
    uint32_t mph = 0;  // UMMA barrier phase
    bool ok = true;

    auto sync_wg = [&]() { named_bar_sync(1, kCompute); };
    // thread 0 waits, then the warpgroup learns the outcome (uniform abort decision)
    auto wg_wait = [&](uint64_t* bar, uint32_t par) -> bool {
      if (tid == 0) wait_bounded(bar, par, m, limit, p.error_word);
      sync_wg();
      return *(volatile int32_t*)&m->abort == 0;
    };
    auto mma_commit_wait = [&]() -> bool {
      if (tid == 0) umma_commit(&m->mma);
      const bool r = wg_wait(&m->mma, mph & 1u);
      ++mph;
      tc_fence_after();
      return r;
    };

    for (int j = 0; j < nchunks && ok; ++j) {
      const int L = min(C, seg.len - j * C);
      const int32_t tok = seg.tok0 + j * C;
      const uint32_t par = (uint32_t)(j & 1);
      if (tid < C) {
        float b = 0.f;
        if (tid < L) b = to_f32(static_cast<const __nv_bfloat16*>(p.beta)[(size_t)(tok + tid) * H + h]);
        m->beta[tid] = b;
      }
      if (!wg_wait(&m->full_qkg, par)) { ok = false; break; }

      // ---------------------------------------------------------------- prep 1: Gram operands
      float gam[32][2];
      {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * hh + i;
          float2 gv = make_float2(0.f, 0.f);
          if (t < L) {
            gv = bf2_to_f2(ld_u32(sm, OFF_G + sw128_off(t, c0, 8192)));
            if (checked && !(gv.x >= KDA_G_MIN && gv.x <= 0.f && gv.y >= KDA_G_MIN && gv.y <= 0.f))
              report_error(p.error_word, KDA_ERR_DECAY_OUT_OF_RANGE);
          }
          a0 += gv.x * kLog2e; a1 += gv.y * kLog2e;
          gam[i][0] = a0; gam[i][1] = a1;
        }
        if (hh == 0) m->tot[pr] = make_float2(a0, a1);
      }
      sync_wg();
      if (hh == 1) {
        const float2 o = m->tot[pr];
#pragma unroll
        for (int i = 0; i < 32; ++i) { gam[i][0] += o.x; gam[i][1] += o.y; }
        m->ref[3][c0] = gam[15][0]; m->ref[3][c0 + 1] = gam[15][1];
        m->ref[4][c0] = gam[31][0]; m->ref[4][c0 + 1] = gam[31][1];
      } else {
        m->ref[0][c0] = 0.f; m->ref[0][c0 + 1] = 0.f;
        m->ref[1][c0] = gam[15][0]; m->ref[1][c0 + 1] = gam[15][1];
        m->ref[2][c0] = gam[31][0]; m->ref[2][c0 + 1] = gam[31][1];
      }
      sync_wg();
      {
        float r[4][2];
#pragma unroll
        for (int a = 0; a < 4; ++a) { r[a][0] = m->ref[a][c0]; r[a][1] = m->ref[a][c0 + 1]; }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * hh + i;
          const int b = t >> 4;  // = 2 hh + (i >> 4)
          float2 kv = make_float2(0.f, 0.f), qv = kv;
          if (t < L) {
            kv = bf2_to_f2(ld_u32(sm, OFF_K + sw128_off(t, c0, 8192)));
            qv = bf2_to_f2(ld_u32(sm, OFF_Q + sw128_off(t, c0, 8192)));
          }
          const float x0 = ex2(gam[i][0] - r[b][0]), x1 = ex2(gam[i][1] - r[b][1]);
          const float ix0 = ex2(r[b][0] - gam[i][0]), ix1 = ex2(r[b][1] - gam[i][1]);
          st_u32(R, R_KQ + sw128_off(t, c0, 16384), f2_to_bf2(kv.x * x0, kv.y * x1));
          st_u32(R, R_KQ + sw128_off(64 + t, c0, 16384), f2_to_bf2(qv.x * x0, qv.y * x1));
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            if (a >= b) {
              const float f0 = ix0 * ex2(r[a][0] - r[b][0]), f1 = ix1 * ex2(r[a][1] - r[b][1]);
              st_u32(R, r_kc(a) + sw128_off(t, c0, 16 * (a + 1) * 128), f2_to_bf2(kv.x * f0, kv.y * f1));
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      sync_wg();
      // ---------------------------------------------------------------- UMMA: A | P
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const uint32_t n = 16u * (a + 1);
          umma_k_loop(tmem + TM_AP + ap_off(a), sm_u + OFF_R + R_KQ, 16, true, 16384, sm_u + OFF_R + r_kc(a), 16,
                      true, n * 128u, 8, idesc_bf16_f32(128, n, 0, 0), false);
        }
      }
      if (!mma_commit_wait()) { ok = false; break; }

      // ---------------------------------------------------------------- read A (beta-scaled) and P
      {
        float* Af = reinterpret_cast<float*>(R + R_AF);
        const int wq = warp & 1;            // subtiles 2wq, 2wq+1 of this warp's 32 rows
        const bool isP = warp >= 2;
        const int t = (warp & 1) * 32 + lane;  // row within A or P
        const float bt = m->beta[t];
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int as = 0; as < 2; ++as) {
          const int a = 2 * wq + as;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            if (kb <= a) {
              uint32_t v[16];
              tmem_ld16(lane_base + TM_AP + ap_off(a) + 16 * kb, v);
              tmem_wait_ld();
              if ((t >> 4) == a) {
                if (!isP) {
#pragma unroll
                  for (int jj = 0; jj < 16; ++jj) {
                    const int s = 16 * kb + jj;
                    Af[t * LDF + s] = (s < t) ? bt * __uint_as_float(v[jj]) : 0.f;
                  }
                } else {
#pragma unroll
                  for (int jj = 0; jj < 16; jj += 2) {
                    const int s = 16 * kb + jj;
                    const float p0 = (s <= t) ? __uint_as_float(v[jj]) : 0.f;
                    const float p1 = (s + 1 <= t) ? __uint_as_float(v[jj + 1]) : 0.f;
                    st_u32(R, R_P + sw128_off(t, s, 8192), f2_to_bf2(p0, p1));
                  }
                }
              }
            }
          }
        }
        if (isP) {  // columns past the row's sub-tile are zero
#pragma unroll
          for (int s = 0; s < C; s += 2)
            if (s >= 16 * ((t >> 4) + 1)) st_u32(R, R_P + sw128_off(t, s, 8192), 0u);
        }
      }
      tc_fence_before();
      sync_wg();

      // ---------------------------------------------------------------- UT inverse
      {
        const float* Lf = reinterpret_cast<const float*>(R + R_AF);
        float* Tf = reinterpret_cast<float*>(R + R_TF);
        float* Y = reinterpret_cast<float*>(R + R_Y);
        if (tid < 64) {  // diagonal 16x16 blocks by forward substitution, one column per thread
          const int a = tid >> 4, jc = tid & 15, o = 16 * a;
          float col[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) col[i] = (i == jc) ? 1.f : 0.f;
#pragma unroll
          for (int i = 1; i < 16; ++i) {
            if (i > jc) {
              float acc = 0.f;
#pragma unroll
              for (int mm = 0; mm < 16; ++mm)
                if (mm < i && mm >= jc) acc += Lf[(o + i) * LDF + o + mm] * col[mm];
              col[i] = -acc;
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) Tf[(o + i) * LDF + o + jc] = col[i];
        }
        sync_wg();
        for (int d = 1; d <= 3; ++d) {  // off-diagonal blocks at distance d
          const int nel = (4 - d) * 256;
          for (int e = tid; e < nel; e += kCompute) {
            const int b = e >> 8, i = (e >> 4) & 15, jc = e & 15, a = b + d;
            float acc = 0.f;
            for (int cc = 16 * b; cc < 16 * a; ++cc) acc += Lf[(16 * a + i) * LDF + cc] * Tf[cc * LDF + 16 * b + jc];
            Y[e] = acc;
          }
          sync_wg();
          for (int e = tid; e < nel; e += kCompute) {
            const int b = e >> 8, i = (e >> 4) & 15, jc = e & 15, a = b + d;
            float acc = 0.f;
            for (int kk = 0; kk <= i; ++kk) acc += Tf[(16 * a + i) * LDF + 16 * a + kk] * Y[(b << 8) + (kk << 4) + jc];
            Tf[(16 * a + i) * LDF + 16 * b + jc] = -acc;
          }
          sync_wg();
        }
        // T' = T Diag(beta), bf16, K-major [64 rows][64]
        for (int e = tid; e < C * C / 2; e += kCompute) {
          const int i = e >> 5, jc = (e & 31) * 2;
          const float t0 = (jc <= i) ? Tf[i * LDF + jc] * m->beta[jc] : 0.f;
          const float t1 = (jc + 1 <= i) ? Tf[i * LDF + jc + 1] * m->beta[jc + 1] : 0.f;
          st_u32(R, R_TP + sw128_off(i, jc, 8192), f2_to_bf2(t0, t1));
        }
      }
      sync_wg();

      // ---------------------------------------------------------------- prep 2: e^g k, e^g q, e^{gC-g} k
      {
        float a0 = 0.f, a1 = 0.f;
        if (hh == 1) { const float2 o = m->tot[pr]; a0 = o.x; a1 = o.y; }
        const float gc0 = m->ref[4][c0], gc1 = m->ref[4][c0 + 1];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * hh + i;
          float2 kv = make_float2(0.f, 0.f), qv = kv, gv = kv;
          if (t < L) {
            gv = bf2_to_f2(ld_u32(sm, OFF_G + sw128_off(t, c0, 8192)));
            kv = bf2_to_f2(ld_u32(sm, OFF_K + sw128_off(t, c0, 8192)));
            qv = bf2_to_f2(ld_u32(sm, OFF_Q + sw128_off(t, c0, 8192)));
          }
          a0 += gv.x * kLog2e; a1 += gv.y * kLog2e;
          const float e0 = ex2(a0), e1 = ex2(a1);
          const float h0 = ex2(gc0 - a0), h1 = ex2(gc1 - a1);
          const uint32_t off = sw128_off(t, c0, 8192);
          st_u32(R, R_KT + off, f2_to_bf2(kv.x * e0, kv.y * e1));
          st_u32(R, R_QT + off, f2_to_bf2(qv.x * e0, qv.y * e1));
          st_u32(R, R_KH + off, f2_to_bf2(kv.x * h0, kv.y * h1));
        }
        if (hh == 0) { m->ec[c0] = ex2(gc0); m->ec[c0 + 1] = ex2(gc1); }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      sync_wg();
      // q, k, g consumed: let the producer fetch the next chunk's tiles
      if (tid == 0) mbar_arrive(&m->empty_qkg);
      // ---------------------------------------------------------------- UMMA: W = T' Kt, U' = T' V
      if (tid == 0) wait_bounded(&m->full_v, par, m, limit, p.error_word);
      sync_wg();
      if (*(volatile int32_t*)&m->abort) { ok = false; break; }
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(64, 128, 0, 1);
        umma_k_loop(tmem + TM_WU, sm_u + OFF_R + R_TP, 16, true, 0, sm_u + OFF_R + R_KT, 8192, false, 0, 4, id,
                    false);
        umma_k_loop(tmem + TM_WU + (16u << 16), sm_u + OFF_R + R_TP, 16, true, 0, sm_u + OFF_V, 8192, false, 0, 4,
                    id, false);
      }
      if (!mma_commit_wait()) { ok = false; break; }
      if (tid == 0) mbar_arrive(&m->empty_v);

      // ---------------------------------------------------------------- -W -> bf16 (rows of the lane-0 tile)
      {
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        const int t = 16 * warp + lane;  // valid for lane < 16
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld32(lane_base + TM_WU + 32 * cb, v);
          tmem_wait_ld();
          if (lane < 16) {
#pragma unroll
            for (int jj = 0; jj < 32; jj += 2)
              st_u32(R, R_W + sw128_off(t, 32 * cb + jj, 8192),
                     f2_to_bf2(-__uint_as_float(v[jj]), -__uint_as_float(v[jj + 1])));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      sync_wg();
      // ---------------------------------------------------------------- UMMA: U = U' - W S0 ; O = Qt S0
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(64, 128, 0, 1);
        umma_k_loop(tmem + TM_WU + (16u << 16), sm_u + OFF_R + R_W, 16, true, 8192, sm_u + OFF_S, 16384, false, 0,
                    8, id, true);
        umma_k_loop(tmem + TM_WU, sm_u + OFF_R + R_QT, 16, true, 8192, sm_u + OFF_S, 16384, false, 0, 8, id, false);
      }
      if (!mma_commit_wait()) { ok = false; break; }

      // ---------------------------------------------------------------- U -> bf16 (rows of the lane-16 tile)
      {
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        const int t = 16 * warp + (lane - 16);  // valid for lane >= 16
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld32(lane_base + TM_WU + 32 * cb, v);
          tmem_wait_ld();
          if (lane >= 16) {
#pragma unroll
            for (int jj = 0; jj < 32; jj += 2)
              st_u32(R, R_U + sw128_off(t, 32 * cb + jj, 8192),
                     f2_to_bf2(__uint_as_float(v[jj]), __uint_as_float(v[jj + 1])));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      sync_wg();
      // ---------------------------------------------------------------- UMMA: O += P U ; K^T U
      if (tid == 0) {
        tc_fence_after();
        umma_k_loop(tmem + TM_WU, sm_u + OFF_R + R_P, 16, true, 0, sm_u + OFF_R + R_U, 8192, false, 0, 4,
                    idesc_bf16_f32(64, 128, 0, 1), true);
        umma_k_loop(tmem + TM_KU, sm_u + OFF_R + R_KH, 8192, false, 0, sm_u + OFF_R + R_U, 8192, false, 0, 4,
                    idesc_bf16_f32(128, 128, 1, 1), false);
      }
      if (!mma_commit_wait()) { ok = false; break; }

      // ---------------------------------------------------------------- state carry
      {
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        const float ec = m->ec[tid];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld32(lane_base + TM_KU + 32 * cb, v);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) S[32 * cb + jj] = ec * S[32 * cb + jj] + __uint_as_float(v[jj]);
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2)
            st_u32(sm, OFF_S + sw128_off(tid, 32 * cb + jj, 16384), f2_to_bf2(S[32 * cb + jj], S[32 * cb + jj + 1]));
        }
      }
      // ---------------------------------------------------------------- epilogue
      if (write_out) {
        if (has_gate && tid == 0) wait_bounded(&m->full_gate, par, m, limit, p.error_word);
        if (has_gate) sync_wg();
        const bool gate_ok = *(volatile int32_t*)&m->abort == 0;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        const int t = 16 * warp + lane;  // O rows: lanes < 16
        float ss = 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld32(lane_base + TM_WU + 32 * cb, v);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) { const float o = __uint_as_float(v[jj]) * p.scale; ss += o * o; }
        }
        const float rr = has_gate ? rsqrtf(ss / (float)DV + p.eps) : 1.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + ((size_t)(tok + t) * H + h) * DV;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld32(lane_base + TM_WU + 32 * cb, v);
          tmem_wait_ld();
          if (lane < 16 && t < L && gate_ok) {
#pragma unroll
            for (int jj = 0; jj < 32; jj += 8) {
              const int c = 32 * cb + jj;
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] = __uint_as_float(v[jj + e]) * p.scale * rr;
              if (has_gate) {
                const uint4 gq = *reinterpret_cast<const uint4*>(sm + OFF_GATE + sw128_off(t, c, 8192));
                const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 gl = bf2_to_f2(gw[e]);
                  const float w0 = p.norm_weight ? __ldg(p.norm_weight + c + 2 * e) : 1.f;
                  const float w1 = p.norm_weight ? __ldg(p.norm_weight + c + 2 * e + 1) : 1.f;
                  y[2 * e] *= w0 / (1.f + __expf(-gl.x));
                  y[2 * e + 1] *= w1 / (1.f + __expf(-gl.y));
                }
              }
              uint4 o;
              o.x = f2_to_bf2(y[0], y[1]); o.y = f2_to_bf2(y[2], y[3]);
              o.z = f2_to_bf2(y[4], y[5]); o.w = f2_to_bf2(y[6], y[7]);
              *reinterpret_cast<uint4*>(orow + c) = o;
            }
          }
        }
      } else if (has_gate) {
        if (tid == 0) wait_bounded(&m->full_gate, par, m, limit, p.error_word);
      }
      tc_fence_before();
      sync_wg();
      if (*(volatile int32_t*)&m->abort) { ok = false; break; }
      if (tid == 0 && has_gate) mbar_arrive(&m->empty_gate);
      fence_proxy_async_smem();  // the bf16 state copy feeds the next chunk's UMMAs
    }

    // ---------------------------------------------------------------- end state
    if (ok) {
      float* dst = nullptr;
      if (seg.role == kRoleWhole || seg.role == kRoleFromWs) {
        if (seg.last && p.final_state) dst = p.final_state + ((size_t)seg.seq * H + h) * unit_state;
      } else if (seg.role == kRoleHead) {
        dst = p.ws_state + ((size_t)(seg.slot + 1) * H + h) * unit_state;
      }
      if (dst) {
#pragma unroll
        for (int c = 0; c < DV; c += 4)
          *reinterpret_cast<float4*>(dst + (size_t)tid * DV + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
      }
    } else if (tid == 0 && mph > 0) {
      // an aborted UMMA group may still be running: wait for it before freeing TMEM
      wait_bounded(&m->mma, (mph - 1) & 1u, m, drain_limit, p.error_word, false);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [T_tot, H, 128] bf16 viewed as 3-D (d, H, T_tot); box (64, 1, 64), 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int H, int64_t T_tot) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)(T_tot > 0 ? T_tot : 1)};
  const cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const Plan& plan, const ChunkParams& p, cudaStream_t stream) {
  if (plan.n_seg == 0) return cudaSuccess;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  const int64_t T = p.total_tokens;
  if (!make_map(&maps.q, p.q, p.H, T) || !make_map(&maps.k, p.k, p.H, T) || !make_map(&maps.g, p.g, p.H, T) ||
      !make_map(&maps.v, p.v, p.H, T))
    return cudaErrorInvalidValue;
  if (p.gate && !make_map(&maps.gate, p.gate, p.H, T)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  chunk_tc_kernel<<<plan.n_seg * plan.H, kThreads, SMEM_BYTES, stream>>>(plan, maps, p);
  return cudaGetLastError();
}

}  // namespace kda
