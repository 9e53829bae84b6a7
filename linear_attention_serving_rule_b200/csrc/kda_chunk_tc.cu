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
// Work split (320 threads): warp 8 is the TMA producer with four groups of tiles: g (with beta,
// handed back right after the decay scan), k and q (landing interleaved as one 128-row tile, each
// with its own barrier: k is handed back after the W|U' UMMAs, q after the U/O UMMAs that read
// its in-place product) and v (after W|U'); it also prefetches each chunk's k, q and v tiles into
// L2 about a chunk ahead.  Warps 0-7
// are two compute warpgroups; warp w owns TMEM lane quarter w % 4.  Decay prep, Gram read-out,
// UT inverse and the -W / U conversions run on all 256 threads; in the shadow of the Gram and of
// the W|U' UMMAs both warpgroups run the previous chunk's epilogue; while warps 0-1 invert the
// diagonal blocks of the UT transform, warps 2-7 make the bf16 copy of the state; in the shadow
// of the U and O UMMAs all warps decay the state and scan the next chunk's decay.  Off-diagonal
// blocks of the inverse are warp-level tf32 MMAs.  Warp 9 issues the UMMAs: the compute warps
// publish each group's operands on an mbarrier and go on with the work beside it.  The gate
// logits are staged from global memory with cp.async into their own buffer.
//
// TMEM (512 columns allocated): [0,128) the fp32 state S (M=128; decayed in place while the
// U and O UMMAs run, then K^T U accumulated onto it); [128,288) A|P (M=128, N=160);
// [288,352) W, [352,416) U' -> U and [416,480) O: each M=64 product is issued as two N=64 halves,
// columns 0-63 at lane offset 0 and columns 64-127 at lane offset 16 of the same TMEM columns, so
// a warp's 32 lanes read 16 rows x 2 column halves and every lane takes part in the read-outs.
// O keeps its own columns so that a chunk's epilogue can run beside the next chunk's UMMAs.
//
// The split's pass 1 (a middle segment's local state and transition matrix, no outputs) runs a
// second copy of the same body on the augmented state [S | M]: no q tile, no P, and the output
// chains replaced by M's (U_M = -W M, M += Kh^T U_M); its TMEM and shared-memory map is given
// beside the layout constants below.
//
// Every wait is bounded (%globaltimer): on expiry the kernel records KDA_ERR_TIMEOUT, stops
// issuing work, drains its own in-flight TMA and UMMA operations (bounded again), frees TMEM
// and returns.
#include <cuda.h>
#include <cstddef>

#include "kda_internal.cuh"
#include "ptx_sm100.cuh"

namespace kda {
namespace {

using namespace ptx;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int kCompute = 256;
constexpr int kThreads = 320;  // 8 compute warps, the TMA producer (warp 8), the UMMA issuer (warp 9)
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;       // k rows 0-63 | q rows 64-127 (TMA); later e^{gamma} k | e^{gamma} q in place
constexpr uint32_t OFF_G = 32768;    // g (TMA)
constexpr uint32_t OFF_V = 49152;    // v (TMA), B operand of U' = T' V
constexpr uint32_t OFF_KC = 65536;   // stacked Kc_0..Kc_3 (160 rows, 40 KB); then fp32 A and T of the inverse
constexpr uint32_t OFF_KL = 106496;  // [k; q] e^{gamma - r_own} (128 rows, 32 KB); then -W; then U
constexpr uint32_t OFF_KH = 139264;  // e^{gamma_C - gamma} k
constexpr uint32_t OFF_S = 155648;   // bf16 state, MN-major [dk rows][dv], two 16 KB column blocks
constexpr uint32_t OFF_TP = 188416;  // T' = T Diag(beta), bf16 [64][64]
constexpr uint32_t OFF_P = 196608;   // P (causally masked), bf16 [64][64]
constexpr uint32_t OFF_MISC = 204800;
constexpr uint32_t OFF_GATE = OFF_MISC + 8192;  // gate logits of the chunk whose epilogue is pending (TMA)
constexpr uint32_t SMEM_BYTES = OFF_GATE + 16384 + 1024;
static_assert(SMEM_BYTES <= 232448, "over the 227 KB of shared memory a block may use");
// fp32 L = Diag(beta) A [64][68], then fp32 T [64][68]: a row stride of 4 mod 32 words keeps the
// mma.sync A-fragment loads (8 rows x 4 columns per warp) free of bank conflicts
constexpr int LDF = 68;
constexpr int LDT = 68;
constexpr uint32_t OFF_TF = OFF_KC + 64 * LDF * 4;

constexpr uint32_t TM_S = 0, TM_AP = 128, TM_WU = 288, TM_O = 416;
// The split's pass 1 runs on the augmented state [S | M] (S from 0 with the values, M from I
// with values 0, so it ends as the segment's transition matrix) and writes no outputs. Its TMEM:
// [0,128) S, [128,256) M, [256,416) A|P; once A is read out, W|U' over [256,384) and U_M = -W M
// in [384,448). Its shared memory reuses what the outputs would take: M's bf16 copy (the B
// operand of -W M) in the gate buffer and in the second column block of the [k; q] tile, which is
// free once the Gram is done; U_M in bf16 over T' and P, free once the W|U' UMMAs are done.
constexpr uint32_t TM_M = 128, TM_AP_AUG = 256, TM_WU_AUG = 256, TM_UM = 384;
constexpr uint32_t OFF_MC0 = OFF_GATE, OFF_MC1 = OFF_KL + 16384, OFF_UM = OFF_TP;
static_assert(OFF_TP + 8192 == OFF_P, "U_M's two column blocks sit over T' and P, 8 KB apart");
static_assert(OFF_MC0 % 1024 == 0 && OFF_MC1 % 1024 == 0, "swizzle atoms need 1024-byte alignment");

// The column operands Kc_0..Kc_3 (16(a+1) rows each) are stacked into one 160-row K-major tile
// (two 64-column blocks of 160 x 128 bytes); Kc_a starts at row ap_off(a), which is also the
// TMEM column offset of sub-tile a's block of A|P, so one N=160 UMMA produces all of A|P.
__host__ __device__ constexpr uint32_t ap_off(int a) { return a == 0 ? 0u : a == 1 ? 16u : a == 2 ? 48u : 96u; }
constexpr uint32_t KC_ROWS = 160, KC_BLK = KC_ROWS * 128;

struct Misc {
  // k and q have their own barriers: the k rows are free after the W|U' UMMAs, the q rows only
  // after the U/O UMMAs
  uint64_t full_g, full_k, full_q, full_v, empty_g, empty_k, empty_q, empty_v, mma, ops;
  uint64_t full_gate, empty_gate;  // the gate tile: loaded per chunk, freed after its epilogue
  uint32_t tmem_base;
  int32_t abort;
  float beta[2][C];  // double-buffered by chunk parity (written by the producer warp)
  float se[4][DK];  // e^{decay over sub-tile m}; channel 8o + e at [m][16 e + o]
  float ec[DK];     // e^{gamma_C}
  alignas(16) float nw[DV];  // RMSNorm weight (1 without one); read as float4
  float ssq[2][C];  // epilogue: per-row sums of squares of the two column halves
  float qkss[2][2 * C];  // with KDA_FLAG_QK_L2NORM: sums of squares of the k|q rows, by column half
};
static_assert(sizeof(Misc) <= 8192, "misc block too large");
static_assert(offsetof(Misc, nw) % 16 == 0, "float4 reads of the norm weight need 16-byte alignment");
static_assert(offsetof(Misc, full_g) % 8 == 0, "mbarriers need 8-byte alignment");

struct TcMaps {
  CUtensorMap q, k, g, v, gate;  // gate: only when the call has gate logits
};
static_assert(sizeof(Plan) + sizeof(TcMaps) + sizeof(ChunkParams) + 128 <= 32764,
              "kernel parameters exceed the 32,764-byte limit");

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
__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
  float2 a = bf2_to_f2(u.x), b = bf2_to_f2(u.y), c = bf2_to_f2(u.z), d = bf2_to_f2(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(f2_to_bf2(f[0], f[1]), f2_to_bf2(f[2], f[3]), f2_to_bf2(f[4], f[5]), f2_to_bf2(f[6], f[7]));
}
// The same 8 values as 4 pairs, for the two-wide fp32 multiply (mul.rn.f32x2: each half rounds
// like mul.rn.f32, so results match the scalar products bit for bit).
__device__ __forceinline__ void unpack8x2(uint4 u, float2 (&f)[4]) {
  f[0] = bf2_to_f2(u.x); f[1] = bf2_to_f2(u.y); f[2] = bf2_to_f2(u.z); f[3] = bf2_to_f2(u.w);
}
__device__ __forceinline__ uint4 pack8x2(const float2 (&f)[4]) {
  return make_uint4(f2_to_bf2(f[0].x, f[0].y), f2_to_bf2(f[1].x, f[1].y), f2_to_bf2(f[2].x, f[2].y),
                    f2_to_bf2(f[3].x, f[3].y));
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<const uint64_t*>(&a)),
      "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&r);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint4& at16(uint8_t* base, uint32_t off) { return *reinterpret_cast<uint4*>(base + off); }

// Warp-level m16n8k8 tf32 MMA (fp32 accumulate).  Fragments, with g = lane / 4, t = lane % 4:
// A (16x8): (g, t), (g+8, t), (g, t+4), (g+8, t+4); B (8x8): (t, g), (t+4, g);
// C (16x8): (g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).
__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// d += a b with both operands rounded to tf32 (nearest).  The inverse's off-diagonal blocks only
// feed T' = T Diag(beta), which is rounded to bf16 (8 mantissa bits) for the W|U' UMMAs; tf32 (11
// bits) products leave the output and state errors unchanged (checked against the oracle on the
// chunk model).
__device__ __forceinline__ void mma_1xtf32(float (&d)[4], const float (&a)[4], const float (&b)[2]) {
  uint32_t ah[4], bh[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) ah[i] = tf32_rna(a[i]);
#pragma unroll
  for (int i = 0; i < 2; ++i) bh[i] = tf32_rna(b[i]);
  mma_tf32(d, ah, bh);
}

// One accumulation chain of a UMMA group: destination, descriptors (built once), operand majors
// and 64-column block strides.  K-major operands step 32 bytes per 16-wide K step and jump to their
// second 64-column block (blk bytes away) after 4 steps; MN-major ones step 2048 bytes.  Each K
// step only adds its byte offset / 16 to the start-address field (bits 0-13), which cannot carry
// out for shared-memory addresses.
struct UChain {
  uint32_t d;
  uint64_t a0, b0;
  uint32_t a_blk, b_blk, idesc;
  bool a_kmajor, b_kmajor, accumulate;
};
__device__ __forceinline__ UChain uchain(uint32_t d, uint32_t a_addr, uint32_t a_lbo, bool a_kmajor, uint32_t a_blk,
                                         uint32_t b_addr, uint32_t b_lbo, bool b_kmajor, uint32_t b_blk, uint32_t idesc,
                                         bool accumulate) {
  return UChain{d, smem_desc_sw128(a_addr, a_lbo, 1024), smem_desc_sw128(b_addr, b_lbo, 1024), a_blk, b_blk, idesc,
                a_kmajor, b_kmajor, accumulate};
}
// Issue NC independent chains of `ksteps` K steps each, interleaved step by step: the K steps of one
// chain accumulate into the same TMEM tile and wait for each other, so the other chains' steps
// fill the tensor pipe meanwhile (issued chain after chain, a group runs at about one step per
// pipe latency).
template <int NC>
__device__ __forceinline__ void umma_interleaved(const UChain (&c)[NC], int ksteps) {
#pragma unroll
  for (int k = 0; k < ksteps; ++k) {
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const uint32_t ao = c[i].a_kmajor ? (uint32_t)(k >> 2) * c[i].a_blk + (uint32_t)(k & 3) * 32u : (uint32_t)k * 2048u;
      const uint32_t bo = c[i].b_kmajor ? (uint32_t)(k >> 2) * c[i].b_blk + (uint32_t)(k & 3) * 32u : (uint32_t)k * 2048u;
      umma_bf16(c[i].d, c[i].a0 + (ao >> 4), c[i].b0 + (bo >> 4), c[i].idesc, (c[i].accumulate || k > 0) ? 1u : 0u);
    }
  }
}

template <bool kPre, bool kOut>
__device__ __forceinline__ void chunk_tc_body(const Plan& plan, const TcMaps& maps, const ChunkParams& p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base (swizzle atoms), offset by pointer arithmetic on the __shared__ array so
  // that every access through sm stays a shared-memory access
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Misc* m = reinterpret_cast<Misc*>(sm + OFF_MISC);
  const uint32_t sm_u = smem_u32(sm);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = plan.H;
  const Seg seg = plan.seg[blockIdx.x / H];
  const int h = blockIdx.x % H;
  const bool has_gate = p.gate != nullptr;
  const bool checked = (p.flags & KDA_FLAG_CHECK_DECAY) != 0;
  const bool g_logits = kPre && (p.flags & KDA_FLAG_G_LOGITS) != 0;
  const bool l2norm = kPre && (p.flags & KDA_FLAG_QK_L2NORM) != 0;
  const uint64_t limit = (p.flags & KDA_FLAG_TEST_FORCE_TIMEOUT) ? 0ull : 2000000000ull;  // 2 s
  const uint64_t drain_limit = 2000000000ull;
  const int nchunks = (seg.len + C - 1) / C;
  constexpr uint32_t tm_ap = kOut ? TM_AP : TM_AP_AUG, tm_wu = kOut ? TM_WU : TM_WU_AUG;
  constexpr bool write_out = kOut;
  const bool stage_gate = write_out && has_gate;  // the epilogue needs the chunk's gate logits

  if (tid == 0) {
    mbar_init(&m->full_g, 1); mbar_init(&m->full_k, 1); mbar_init(&m->full_q, 1); mbar_init(&m->full_v, 1);
    mbar_init(&m->empty_g, 1); mbar_init(&m->empty_k, 1); mbar_init(&m->empty_q, 1); mbar_init(&m->empty_v, 1);
    mbar_init(&m->mma, 1);
    mbar_init(&m->full_gate, 1);
    mbar_init(&m->empty_gate, 1);
    mbar_init(&m->ops, 8);  // one arrival per compute warp: a UMMA group's operands are in place
    m->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&m->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.g); prefetch_tmap(&maps.v);
    if (stage_gate) prefetch_tmap(&maps.gate);
  }
  if (tid < DV) m->nw[tid] = p.norm_weight ? p.norm_weight[tid] : 1.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = m->tmem_base;

  if (warp == 8) {
    // ===================================================================== TMA producer
    // Lane 0 issues the tile loads; the whole warp first fetches the chunk's beta into the
    // double buffer m->beta[j & 1], published by the same mbarrier as the g tile.
    int ig = -1, ik = -1, iq = -1, iv = -1, igt = -1;  // last chunk whose g, k, q, v, gate loads were issued
    auto load_gate = [&](int jg) -> bool {  // lane 0
      if (!wait_bounded(&m->empty_gate, (uint32_t)((jg & 1) ^ 1), m, drain_limit, p.error_word)) return false;
      mbar_arrive_expect_tx(&m->full_gate, 16384);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_3d(sm + OFF_GATE + hf * 8192, &maps.gate, &m->full_gate, hf * 64, h, seg.tok0 + jg * C);
      igt = jg;
      return true;
    };
    bool prod_ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int32_t tok = seg.tok0 + j * C;
      const int L = min(C, seg.len - j * C);
      const uint32_t par = (uint32_t)((j & 1) ^ 1);
      // the chunk's k, q and v tiles into L2 now, about a chunk before their buffers free up (the q
      // load is issued only once the previous chunk's U/O UMMAs are done, on the critical path)
      if (lane == 0) {
        for (int hf = 0; hf < 2; ++hf) {
          tma_prefetch_3d(&maps.k, hf * 64, h, tok);
          if (write_out) tma_prefetch_3d(&maps.q, hf * 64, h, tok);
          tma_prefetch_3d(&maps.v, hf * 64, h, tok);
        }
      }
      int okw = 1;
      if (lane == 0) okw = wait_bounded(&m->empty_g, par, m, drain_limit, p.error_word) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = lane + 32 * r;
        float bv = (t < L) ? to_f32(static_cast<const __nv_bfloat16*>(p.beta)[(size_t)(tok + t) * H + h]) : 0.f;
        if ((p.flags & KDA_FLAG_BETA_LOGITS) && t < L) bv = 1.f / (1.f + expf(-bv));  // beta = sigmoid(b)
        m->beta[j & 1][t] = bv;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&m->full_g, 16384);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + OFF_G + hf * 8192, &maps.g, &m->full_g, hf * 64, h, tok);
      }
      ig = j;
      // the previous chunk's gate logits (its epilogue runs beside this chunk's Gram and W|U'
      // UMMAs): the buffer frees once the epilogue of the chunk before it is done, which is when
      // this chunk's k rows free too, so waiting for it here delays nothing
      if (stage_gate && j > 0) {
        if (lane == 0) okw = load_gate(j - 1) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) break;
      }
      if (lane == 0) okw = wait_bounded(&m->empty_k, par, m, drain_limit, p.error_word) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&m->full_k, 16384);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + OFF_KQ + hf * 16384, &maps.k, &m->full_k, hf * 64, h, tok);
      }
      ik = j;
      if (write_out) {  // the split's pass 1 writes no outputs and needs no q
        if (lane == 0) okw = wait_bounded(&m->empty_q, par, m, drain_limit, p.error_word) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&m->full_q, 16384);
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sm + OFF_KQ + hf * 16384 + 8192, &maps.q, &m->full_q, hf * 64, h, tok);
        }
        iq = j;
      }
      if (lane == 0) okw = wait_bounded(&m->empty_v, par, m, drain_limit, p.error_word) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&m->full_v, 16384);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + OFF_V + hf * 8192, &maps.v, &m->full_v, hf * 64, h, tok);
      }
      iv = j;
    }
    prod_ok = *(volatile int32_t*)&m->abort == 0;
    // the last chunk's gate logits
    if (stage_gate && nchunks > 0 && prod_ok && lane == 0) load_gate(nchunks - 1);
    __syncwarp();
    // drain: after an abort, wait (bounded, regardless of the abort) for the loads issued
    if (lane == 0 && *(volatile int32_t*)&m->abort) {
      if (igt >= 0) wait_bounded(&m->full_gate, (uint32_t)(igt & 1), m, drain_limit, p.error_word, false);
      if (ig >= 0) wait_bounded(&m->full_g, (uint32_t)(ig & 1), m, drain_limit, p.error_word, false);
      if (ik >= 0) wait_bounded(&m->full_k, (uint32_t)(ik & 1), m, drain_limit, p.error_word, false);
      if (iq >= 0) wait_bounded(&m->full_q, (uint32_t)(iq & 1), m, drain_limit, p.error_word, false);
      if (iv >= 0) wait_bounded(&m->full_v, (uint32_t)(iv & 1), m, drain_limit, p.error_word, false);
    }
  } else if (warp == 9) {
    // ===================================================================== UMMA issuer
    // Lane 0 issues each UMMA group once the eight compute warps have published its operands
    // (one arrival each on m->ops) and commits it to m->mma.  Issuing blocks for as long as the
    // tensor core takes to accept the group, so the compute warps never issue.
    if (lane == 0) {
      uint32_t oph = 0;
      int committed = 0;
      const uint32_t hi = 16u << 16;
      for (int j = 0; j < nchunks; ++j) {
        const uint32_t par = (uint32_t)(j & 1);
        // A | P over the stacked Kc operand: one N=160 chain.  The issuing thread waits about the
        // same time per K step whatever N is, so one wide chain beats two interleaved N=80 halves
        // (measured 1.6 K against 2.4 K cycles for the group alone).
        if (!wait_bounded(&m->ops, (oph++) & 1u, m, limit, p.error_word)) break;
        tc_fence_after();
        {
          const uint64_t a0 = smem_desc_sw128(sm_u + OFF_KL, 16, 1024), b0 = smem_desc_sw128(sm_u + OFF_KC, 16, 1024);
          const uint32_t id = idesc_bf16_f32(128, KC_ROWS, 0, 0);
#pragma unroll 1
          for (int k = 0; k < 8; ++k)  // (a rolled loop: each step waits ~180 cycles anyway)
            umma_bf16(tmem + tm_ap, a0 + (((k >> 2) * 16384u + (k & 3) * 32u) >> 4),
                      b0 + (((k >> 2) * KC_BLK + (k & 3) * 32u) >> 4), id, k > 0 ? 1u : 0u);
        }
        umma_commit(&m->mma);
        ++committed;
        // W | U': columns 0-63 at lane offset 0, 64-127 at lane offset 16: W in [288,352), U' in
        // [352,416); one N=128 UMMA per half, whose B operand is [e^g k block | v block] -- two MN
        // atoms (OFF_V - OFF_KQ) and (OFF_V + 8192 - OFF_KQ - 16384) bytes apart
        if (!wait_bounded(&m->ops, (oph++) & 1u, m, limit, p.error_word)) break;
        if (!wait_bounded(&m->full_v, par, m, limit, p.error_word)) break;
        tc_fence_after();
        {
          const uint32_t id = idesc_bf16_f32(64, 128, 0, 1);
          const UChain c[2] = {
              uchain(tmem + tm_wu, sm_u + OFF_TP, 16, true, 0, sm_u + OFF_KQ, OFF_V - OFF_KQ, false, 0, id, false),
              uchain(tmem + tm_wu + hi, sm_u + OFF_TP, 16, true, 0, sm_u + OFF_KQ + 16384,
                     OFF_V + 8192 - OFF_KQ - 16384, false, 0, id, false)};
          umma_interleaved(c, 4);
        }
        umma_commit(&m->mma);
        ++committed;
        // U = U' - W S0 ; O = Qt S0  (pass 1: U = U' - W S0 ; U_M = -W M0)
        if (!wait_bounded(&m->ops, (oph++) & 1u, m, limit, p.error_word)) break;
        tc_fence_after();
        {
          const uint32_t id = idesc_bf16_f32(64, 64, 0, 1);
          const UChain cu0 = uchain(tmem + tm_wu + 64, sm_u + OFF_KL, 16, true, 8192, sm_u + OFF_S, 16384, false, 0,
                                    id, true);
          const UChain cu1 = uchain(tmem + tm_wu + 64 + hi, sm_u + OFF_KL, 16, true, 8192, sm_u + OFF_S + 16384,
                                    16384, false, 0, id, true);
          if (kOut) {
            const UChain c[4] = {
                cu0, cu1,
                uchain(tmem + TM_O, sm_u + OFF_KQ + 8192, 16, true, 16384, sm_u + OFF_S, 16384, false, 0, id, false),
                uchain(tmem + TM_O + hi, sm_u + OFF_KQ + 8192, 16, true, 16384, sm_u + OFF_S + 16384, 16384, false, 0,
                       id, false)};
            umma_interleaved(c, 8);
          } else {
            const UChain c[4] = {
                cu0, cu1,
                uchain(tmem + TM_UM, sm_u + OFF_KL, 16, true, 8192, sm_u + OFF_MC0, 16384, false, 0, id, false),
                uchain(tmem + TM_UM + hi, sm_u + OFF_KL, 16, true, 8192, sm_u + OFF_MC1, 16384, false, 0, id, false)};
            umma_interleaved(c, 8);
          }
        }
        umma_commit(&m->mma);
        ++committed;
        // O += P U ; S += Kh^T U  (pass 1: S += Kh^T U ; M += Kh^T U_M)
        if (!wait_bounded(&m->ops, (oph++) & 1u, m, limit, p.error_word)) break;
        tc_fence_after();
        {
          const UChain cs = uchain(tmem + TM_S, sm_u + OFF_KH, 8192, false, 0, sm_u + OFF_KL, 8192, false, 0,
                                   idesc_bf16_f32(128, 128, 1, 1), true);
          if (kOut) {
            const UChain c[3] = {
                uchain(tmem + TM_O, sm_u + OFF_P, 16, true, 0, sm_u + OFF_KL, 8192, false, 0,
                       idesc_bf16_f32(64, 64, 0, 1), true),
                uchain(tmem + TM_O + hi, sm_u + OFF_P, 16, true, 0, sm_u + OFF_KL + 8192, 8192, false, 0,
                       idesc_bf16_f32(64, 64, 0, 1), true),
                cs};
            umma_interleaved(c, 4);
          } else {
            const UChain c[2] = {
                cs, uchain(tmem + TM_M, sm_u + OFF_KH, 8192, false, 0, sm_u + OFF_UM, 8192, false, 0,
                           idesc_bf16_f32(128, 128, 1, 1), true)};
            umma_interleaved(c, 4);
          }
        }
        umma_commit(&m->mma);
        ++committed;
      }
      // the last group committed must finish before TMEM is freed (after an abort too)
      if (committed > 0)
        wait_bounded(&m->mma, (uint32_t)(committed - 1) & 1u, m, drain_limit, p.error_word, false);
    }
    __syncwarp();
  } else {
    // ===================================================================== compute warpgroups
    const int q4 = warp & 3;   // TMEM lane quarter
    const int wg = warp >> 2;  // column half
    const int row = 32 * q4 + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    const size_t unit_state = (size_t)DK * DV;
    // chunk-boundary snapshot of the state after segment-local token e, or null
    auto snap_dst = [&](int e) -> float* {
      if (seg.snap < 0 || e < seg.snap_off || (e - seg.snap_off) % p.snap_interval != 0) return nullptr;
      const int row_s = seg.snap + (e - seg.snap_off) / p.snap_interval;
      return p.snapshots + ((size_t)row_s * H + h) * unit_state;
    };
    uint32_t mph = 0;
    bool ok = true;

    auto sync_wg = [&]() { named_bar_sync(1, kCompute); };
    // thread 0 waits, then both warpgroups learn the outcome (uniform abort decision)
    auto wg_wait = [&](uint64_t* bar, uint32_t par) -> bool {
      if (tid == 0) wait_bounded(bar, par, m, limit, p.error_word);
      sync_wg();
      return *(volatile int32_t*)&m->abort == 0;
    };
    // publish this warp's operand writes (shared memory and TMEM) to the UMMA issuer
    auto ops_arrive = [&]() {
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&m->ops);
    };

    // ---------------------------------------------------------------- start state -> TMEM + bf16 copy
    {
      const float* src = nullptr;
      if (seg.role == kRoleWhole) {
        if (p.initial_state) src = p.initial_state + ((size_t)seg.seq * H + h) * unit_state;
      } else if (seg.role == kRoleFromWs) {
        src = p.ws_state + ((size_t)seg.slot * H + h) * unit_state;
      }
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        const int c0 = wg * 64 + hb * 32;
        uint32_t v[32];
        if (!kOut) {  // pass 1: M = I (its bf16 copy is made per chunk, beside the W|U' UMMAs)
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __float_as_uint(c0 + jj == row ? 1.f : 0.f);
          tmem_st32(tl + TM_M + c0, v);
        }
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4) {
          float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)row * DV + c0 + jj)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
          v[jj] = __float_as_uint(x.x); v[jj + 1] = __float_as_uint(x.y);
          v[jj + 2] = __float_as_uint(x.z); v[jj + 3] = __float_as_uint(x.w);
        }
        tmem_st32(tl + TM_S + c0, v);
#pragma unroll
        for (int oc = 0; oc < 4; ++oc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]);
          at16(sm, OFF_S + sw128_oct(row, (c0 >> 3) + oc, 16384)) = pack8(f);
        }
      }
      tmem_wait_st();
    }

    // The gate logits of a chunk arrive by TMA (128-byte swizzled [64 tokens][128 B] blocks, one
    // per 64 columns) while the next chunk's prep runs; epilogue part A waits for them and the
    // buffer is handed back after part B.
    // Epilogue of one chunk, run by both warpgroups in two parts while the next chunk's UMMAs run:
    // O stays in TMEM columns [416,480) until the next chunk's O UMMAs.  Lanes l < 16 of warp
    // (q, wg) hold columns 32 wg .. 32 wg + 31 and lanes l + 16 columns 64 + 32 wg .. of O row
    // 16 q + l; a row's sum of squares is combined across the two lanes with a shuffle and across
    // the warpgroups through shared memory.  Part A (beside the Gram UMMAs) finds the row scale
    // and writes the thread's first 16 columns, part B (beside the W|U' UMMAs) the other 16.
    float epi_sc = 0.f;  // scale / rms of the thread's O row, from part A to part B
    auto epi_store = [&](int L_e, int32_t tok_e, const uint32_t* v, int oc0) {
      const int t = 16 * q4 + (lane & 15);
      if (t >= L_e) return;
      const int c0 = 64 * (lane >> 4) + 32 * wg;
      uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + ((size_t)(tok_e + t) * H + h) * DV + c0);
#pragma unroll
      for (int oc = 0; oc < 2; ++oc) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]) * epi_sc;
        if (has_gate) {
          float gl8[8];
          const int c16 = (c0 >> 3) + oc0 + oc;
          unpack8(at16(sm, OFF_GATE + sw128_oct(t, c16, 8192)), gl8);
          const float4 w0 = *reinterpret_cast<const float4*>(&m->nw[c0 + 8 * (oc0 + oc)]);
          const float4 w1 = *reinterpret_cast<const float4*>(&m->nw[c0 + 8 * (oc0 + oc) + 4]);
          const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          // sigmoid(x) = (1 + tanh(x / 2)) / 2: one MUFU operation per element
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float hw = 0.5f * w[e] * f[e];
            f[e] = fmaf(hw, tanh_approx(0.5f * gl8[e]), hw);
          }
        }
        op[oc0 + oc] = pack8(f);
      }
    };
    auto epilogue_a = [&](int L_e, int32_t tok_e) {
      const int t = 16 * q4 + (lane & 15);
      uint32_t v[32];
      tmem_ld32(tl + TM_O + 32 * wg, v);
      tmem_wait_ld();
      float ss = 0.f;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const float a0 = __uint_as_float(v[jj]);
        ss += a0 * a0;
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      if (lane < 16) m->ssq[wg][t] = ss;
      sync_wg();
      ss += m->ssq[wg ^ 1][t];
      const float rr = has_gate ? rsqrtf(ss * p.scale * p.scale / (float)DV + p.eps) : 1.f;
      epi_sc = p.scale * rr;
      epi_store(L_e, tok_e, v, 0);
    };
    auto epilogue_b = [&](int L_e, int32_t tok_e) {
      uint32_t v[16];
      tmem_ld16(tl + TM_O + 32 * wg + 16, v);
      tmem_wait_ld();
      epi_store(L_e, tok_e, v, 2);
    };
    // bf16 copy of the state S for the UMMAs: 64-column halves [hb0, hb1) of this warp's 32 rows;
    // with snap != null also the fp32 snapshot of S
    auto state_copy = [&](int hb0, int hb1, float* snap) {
#pragma unroll 1
      for (int hb = hb0; hb < hb1; ++hb) {
        uint32_t v[64];
        tmem_ld32(tl + TM_S + 64 * hb, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tl + TM_S + 64 * hb + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (snap) {
          float4* d4 = reinterpret_cast<float4*>(snap + (size_t)row * DV + 64 * hb);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            d4[jj] = make_float4(__uint_as_float(v[4 * jj]), __uint_as_float(v[4 * jj + 1]),
                                 __uint_as_float(v[4 * jj + 2]), __uint_as_float(v[4 * jj + 3]));
        }
#pragma unroll
        for (int oc = 0; oc < 8; ++oc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]);
          at16(sm, OFF_S + sw128_oct(row, 8 * hb + oc, 16384)) = pack8(f);
        }
      }
    };

    // thread of the decay scan and prep: channels 8o .. 8o+7, tokens t0 .. t0+3 of sub-tile b.
    // Eight consecutive lanes take eight channel octets of one token, so each quarter-warp's
    // 16-byte accesses to a 128-byte swizzled tile hit eight distinct bank groups.
    const int o = (lane & 7) + 8 * (warp & 1), qq = (lane >> 3) & 3, b = tid >> 6;
    const int t0 = 16 * b + 4 * qq;
    // Decay scan of one chunk (L tokens): gl = inclusive cumulative log2-decay from the start of
    // the thread's sub-tile; se[m] = e^{decay over sub-tile m} per channel.
    auto scan = [&](int L, float (&gl)[4][8]) {
      bool bad = false;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = t0 + i;
        float g8[8];
        if (t < L) {
          unpack8(at16(sm, OFF_G + sw128_oct(t, o, 8192)), g8);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) g8[e] = 0.f;
        }
        if (g_logits && t < L) {  // g = g_min sigmoid(a); the exponent is clamped to keep 1 + e finite
#pragma unroll
          for (int e = 0; e < 8; ++e) g8[e] = __fdividef(KDA_G_MIN, 1.f + ex2(fminf(-g8[e] * kLog2e, 126.f)));
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          bad |= !(g8[e] >= KDA_G_MIN && g8[e] <= 0.f);
          acc[e] += g8[e] * kLog2e;
          gl[i][e] = acc[e];
        }
      }
      if (checked && bad) report_error(p.error_word, KDA_ERR_DECAY_OUT_OF_RANGE);
      // prefix over the four threads of the sub-tile (lanes 8 apart)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float x = acc[e];
        float y = __shfl_up_sync(0xffffffffu, x, 8);
        if (qq >= 1) x += y;
        y = __shfl_up_sync(0xffffffffu, x, 16);
        if (qq >= 2) x += y;
        const float excl = x - acc[e];
#pragma unroll
        for (int i = 0; i < 4; ++i) gl[i][e] += excl;
        if (qq == 3) m->se[b][16 * e + o] = ex2(x);  // decay over the whole sub-tile
      }
    };

    int L_prev = 0;
    int32_t tok_prev = 0;
    float gl[4][8];  // the current chunk's decay scan
    if (nchunks > 0) {  // the first chunk's scan; later ones run in the shadow of the previous chunk's UMMAs
      ok = wg_wait(&m->full_g, 0);
      if (ok) {
        scan(min(C, seg.len), gl);
        if (tid == 0) mbar_arrive(&m->empty_g);
      }
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      const int L = min(C, seg.len - j * C);
      const int32_t tok = seg.tok0 + j * C;
      const uint32_t par = (uint32_t)(j & 1);
      const float* beta = m->beta[j & 1];
      // ---------------------------------------------------------------- decay prep: all bf16 operands

      {
        if (tid == 0 && wait_bounded(&m->full_k, par, m, limit, p.error_word) && write_out)
          wait_bounded(&m->full_q, par, m, limit, p.error_word);
        sync_wg();
        if (*(volatile int32_t*)&m->abort != 0) { ok = false; break; }
      }
      if (l2norm) {  // sums of squares of the raw k | q rows (two column halves per row)
        const int rr = tid & 127, hf = tid >> 7;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float f[8];
          unpack8(at16(sm, OFF_KQ + sw128_oct(rr, 8 * hf + i, 16384)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
        }
        m->qkss[hf][rr] = ss;
        sync_wg();
      }
      // Per-channel factors, applied so that no O(1) value is multiplied by an underflowed
      // constant: with se_m = e^{decay over sub-tile m}, Eb = e^{r_b} = prod_{m<b} se_m, and per
      // token ix = e^{r_b - gamma_t} in [1, e^80]; the chain ix, ix se_b, ix se_b se_{b+1}, ...
      // gives e^{r_a - gamma_t} for a = b..3, each factor <= 1 after the first.
      float Eb[8], sb[8];
      {
        float s1[8], s2[8], s3[8];  // se_{b+1}, se_{b+2} (1 past the last sub-tile); se_3
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float se[4];
#pragma unroll
          for (int mm = 0; mm < 4; ++mm) se[mm] = m->se[mm][16 * e + o];
          float eb = 1.f;
#pragma unroll
          for (int mm = 0; mm < 4; ++mm)
            if (mm < b) eb *= se[mm];
          Eb[e] = eb;
          sb[e] = b == 0 ? se[0] : b == 1 ? se[1] : b == 2 ? se[2] : se[3];
          s1[e] = b == 0 ? se[1] : b == 1 ? se[2] : b == 2 ? se[3] : 1.f;
          s2[e] = b == 0 ? se[2] : b == 1 ? se[3] : 1.f;
          s3[e] = se[3];
        }
        float2 Eb2[4], sb2[4], s1_2[4], s2_2[4], s3_2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          Eb2[c] = make_float2(Eb[2 * c], Eb[2 * c + 1]);
          sb2[c] = make_float2(sb[2 * c], sb[2 * c + 1]);
          s1_2[c] = make_float2(s1[2 * c], s1[2 * c + 1]);
          s2_2[c] = make_float2(s2[2 * c], s2[2 * c + 1]);
          s3_2[c] = make_float2(s3[2 * c], s3[2 * c + 1]);
        }
        // channel pairs (2c, 2c+1) as float2 throughout
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = t0 + i;
          float2 kf[4], qf[4], x[4], ix[4], f[4], fq[4];
          if (t < L) {
            unpack8x2(at16(sm, OFF_KQ + sw128_oct(t, o, 16384)), kf);
            if (write_out) {
              unpack8x2(at16(sm, OFF_KQ + sw128_oct(64 + t, o, 16384)), qf);
            } else {  // no q in the split's pass 1: P and O are not needed
#pragma unroll
              for (int c = 0; c < 4; ++c) qf[c] = make_float2(0.f, 0.f);
            }
            if (l2norm) {  // x / sqrt(|x|^2 + eps)
              const float rk = rsqrtf(m->qkss[0][t] + m->qkss[1][t] + KDA_L2NORM_EPS);
              const float rq = write_out ? rsqrtf(m->qkss[0][64 + t] + m->qkss[1][64 + t] + KDA_L2NORM_EPS) : 0.f;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                kf[c] = fmul2(kf[c], make_float2(rk, rk));
                qf[c] = fmul2(qf[c], make_float2(rq, rq));
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) { kf[c] = make_float2(0.f, 0.f); qf[c] = make_float2(0.f, 0.f); }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            x[c] = make_float2(ex2(gl[i][2 * c]), ex2(gl[i][2 * c + 1]));
            ix[c] = make_float2(ex2(-gl[i][2 * c]), ex2(-gl[i][2 * c + 1]));
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) { f[c] = fmul2(kf[c], x[c]); fq[c] = fmul2(qf[c], x[c]); }
          at16(sm, OFF_KL + sw128_oct(t, o, 16384)) = pack8x2(f);
          if (write_out) at16(sm, OFF_KL + sw128_oct(64 + t, o, 16384)) = pack8x2(fq);
          // e^{gamma} k and e^{gamma} q, in place over the raw tiles (this thread's own elements)
#pragma unroll
          for (int c = 0; c < 4; ++c) { f[c] = fmul2(f[c], Eb2[c]); fq[c] = fmul2(fq[c], Eb2[c]); }
          at16(sm, OFF_KQ + sw128_oct(t, o, 16384)) = pack8x2(f);
          if (write_out) at16(sm, OFF_KQ + sw128_oct(64 + t, o, 16384)) = pack8x2(fq);
          // Kc_a = k e^{r_a - gamma_t}: k ix for a = b, then k ix se_b se_{b+1} ... se_{a-1};
          // the last one (a = 3) times se_3 is e^{gamma_C - gamma_t} k, the state-carry operand
#pragma unroll
          for (int c = 0; c < 4; ++c) f[c] = fmul2(kf[c], ix[c]);
          at16(sm, OFF_KC + sw128_oct(ap_off(b) + t, o, KC_BLK)) = pack8x2(f);
          if (b < 3) {
#pragma unroll
            for (int c = 0; c < 4; ++c) f[c] = fmul2(f[c], sb2[c]);
            at16(sm, OFF_KC + sw128_oct(ap_off(b + 1) + t, o, KC_BLK)) = pack8x2(f);
            if (b < 2) {
#pragma unroll
              for (int c = 0; c < 4; ++c) f[c] = fmul2(f[c], s1_2[c]);
              at16(sm, OFF_KC + sw128_oct(ap_off(b + 2) + t, o, KC_BLK)) = pack8x2(f);
              if (b < 1) {
#pragma unroll
                for (int c = 0; c < 4; ++c) f[c] = fmul2(f[c], s2_2[c]);
                at16(sm, OFF_KC + sw128_oct(ap_off(3) + t, o, KC_BLK)) = pack8x2(f);
              }
            }
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) f[c] = fmul2(f[c], s3_2[c]);
          at16(sm, OFF_KH + sw128_oct(t, o, 8192)) = pack8x2(f);
        }
      }
      if (tid < DK) {
        const int si = 16 * (tid & 7) + (tid >> 3);
        m->ec[tid] = m->se[0][si] * m->se[1][si] * m->se[2][si] * m->se[3][si];
      }
      ops_arrive();  // ---------------------------------------------- UMMA: A | P (issued by warp 9)
      // ---------------------------------------------------------------- in the shadow of the Gram UMMAs:
      // the previous chunk's epilogue (its O is still in TMEM)
      if (write_out && j > 0) {
        if (stage_gate && !wg_wait(&m->full_gate, (uint32_t)((j - 1) & 1))) { ok = false; break; }
        epilogue_a(L_prev, tok_prev);
      }
      {
        const bool r = wg_wait(&m->mma, mph & 1u);
        ++mph;
        tc_fence_after();
        if (!r) { ok = false; break; }
      }

      // ---------------------------------------------------------------- read A (beta-scaled) and P
      {
        float* Af = reinterpret_cast<float*>(sm + OFF_KC);
        const bool isP = q4 >= 2;
        const int t = (q4 & 1) * 32 + lane;
        const int a = 2 * (q4 & 1) + wg;  // the sub-tile whose columns this warp loads
        const bool mine = (t >> 4) == a;
        const float bt = beta[t];
        // the warp's column blocks two at a time: both loads in flight, then one wait
#pragma unroll
        for (int kp = 0; kp < 4; kp += 2) {
          if (kp > a) break;
          uint32_t v[2][16];
          tmem_ld16(tl + tm_ap + ap_off(a) + 16 * kp, v[0]);
          if (kp + 1 <= a) tmem_ld16(tl + tm_ap + ap_off(a) + 16 * (kp + 1), v[1]);
          tmem_wait_ld();
          if (mine && (write_out || !isP)) {  // (P only where outputs are written)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int kb = kp + h2;
              if (kb > a) break;
              if (!isP) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                  const int s = 16 * kb + 4 * c4;
                  const uint32_t* w = &v[h2][4 * c4];
                  *reinterpret_cast<float4*>(&Af[t * LDF + s]) = make_float4(
                      s < t ? bt * __uint_as_float(w[0]) : 0.f, s + 1 < t ? bt * __uint_as_float(w[1]) : 0.f,
                      s + 2 < t ? bt * __uint_as_float(w[2]) : 0.f, s + 3 < t ? bt * __uint_as_float(w[3]) : 0.f);
                }
              } else {
#pragma unroll
                for (int oc = 0; oc < 2; ++oc) {
                  float f[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    f[e] = (16 * kb + 8 * oc + e <= t) ? __uint_as_float(v[h2][8 * oc + e]) : 0.f;
                  at16(sm, OFF_P + sw128_oct(t, 2 * kb + oc, 8192)) = pack8(f);
                }
              }
            }
          }
        }
        if (isP && mine && write_out) {
#pragma unroll
          for (int oc = 0; oc < 8; ++oc)
            if (oc >= 2 * (a + 1)) at16(sm, OFF_P + sw128_oct(t, oc, 8192)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      sync_wg();
      // ---------------------------------------------------------------- UT inverse: T' = (I + Diag(beta) A)^-1 Diag(beta)
      // L = Diag(beta) A (strictly lower).  Diagonal 16x16 blocks of T by forward substitution
      // (one column per thread), then the off-diagonal blocks by block distance d:
      //   T_ab = -T_aa sum_{c in blocks b..a-1} L_{a c} T_{c b},  a = b + d.
      {
        const float* Lf = reinterpret_cast<const float*>(sm + OFF_KC);
        float* Tf = reinterpret_cast<float*>(sm + OFF_TF);
        if (tid < 64) {
          const int a = tid >> 4, jc = tid & 15, o = 16 * a;
          float col[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) col[i] = (i == jc) ? 1.f : 0.f;
#pragma unroll
          for (int i = 1; i < 16; ++i) {
            const float* lr = Lf + (o + i) * LDF + o;
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int mm = 0; mm < i; ++mm) s4[mm & 3] += lr[mm] * col[mm];  // col[mm] = 0 for mm < jc
            const float acc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            col[i] = (i == jc) ? 1.f : (i > jc ? -acc : 0.f);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) Tf[(o + i) * LDT + o + jc] = col[i];
        } else {
          // meanwhile warps 2-7 make the bf16 copy of the state: warps 4 and 5 own TMEM lane
          // quarters 0 and 1 alone, warps 2|6 and 3|7 share quarters 2 and 3
          // (the state here is the one after the previous chunk: a snapshot if that chunk ended
          // on a snapshot boundary)
          float* snap = j > 0 ? snap_dst(j * C) : nullptr;
          if (q4 < 2) state_copy(0, 2, snap);
          else state_copy(warp < 4 ? 0 : 1, warp < 4 ? 1 : 2, snap);
        }
        sync_wg();
        // T' = T Diag(beta) in bf16, item idx = row i, column octet oc (T is zero above the diagonal)
        auto pack_tp = [&](int idx) {
          const int i = idx >> 3, oc = idx & 7;
          const float4 t0 = *reinterpret_cast<const float4*>(Tf + i * LDT + 8 * oc);
          const float4 t1 = *reinterpret_cast<const float4*>(Tf + i * LDT + 8 * oc + 4);
          const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int jc = 8 * oc + e;
            f[e] = (jc <= i) ? tv[e] * beta[jc] : 0.f;
          }
          at16(sm, OFF_TP + sw128_oct(i, oc, 8192)) = pack8(f);
        };
        // Off-diagonal blocks level by level (block distance d), one 16x8 strip per warp: warp
        // w < 2 (4 - d) takes a = b + d with b = w / 2 and columns 16 b + 8 (w % 2) .. +7:
        //   Y = sum_{c=b}^{a-1} L_ac T_cb,   T_ab = -T_aa Y,
        // as m16n8k8 tf32 MMAs.  Y never leaves the warp: its C fragment becomes the B fragment
        // of the second product by shuffles.  A level reads only blocks of earlier levels.  The
        // warps a level leaves idle pack the row blocks of T' that are final: rows 0-15 (final
        // after the diagonal blocks) beside level 1, rows 16-31 beside level 2, rows 32-47 beside
        // level 3; rows 48-63 follow the last level.
        {
          const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
          for (int d = 1; d <= 3; ++d) {
            if (warp < 2 * (4 - d)) {
              const int b = warp >> 1, n0 = 8 * (warp & 1), a = b + d;
              float acc[2][4];  // by K-step parity: two independent chains
#pragma unroll
              for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[u][i] = 0.f;
              const float* la = Lf + (16 * a + g) * LDF + t4;
              const float* tb = Tf + t4 * LDT + 16 * b + n0 + g;
#pragma unroll
              for (int ks = 0; ks < 2 * d; ++ks) {
                const int kk = 16 * b + 8 * ks;
                const float af[4] = {la[kk], la[8 * LDF + kk], la[kk + 4], la[8 * LDF + kk + 4]};
                const float bf[2] = {tb[kk * LDT], tb[(kk + 4) * LDT]};
                mma_1xtf32(acc[ks & 1], af, bf);
              }
              float y[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) y[i] = acc[0][i] + acc[1][i];
              // Y[r][n] sits in lane 4 (r % 8) + n / 2, register 2 (r / 8) + n % 2; this lane needs
              // Y[t][g], Y[t+4][g] (first K step) and Y[8+t][g], Y[12+t][g] (second)
              const int s0 = 4 * t4 + (g >> 1), s1 = s0 + 16;
              const bool odd = (g & 1) != 0;
              float yb[4];
              {
                const float u0 = __shfl_sync(0xffffffffu, y[0], s0), v0 = __shfl_sync(0xffffffffu, y[1], s0);
                const float u1 = __shfl_sync(0xffffffffu, y[0], s1), v1 = __shfl_sync(0xffffffffu, y[1], s1);
                const float u2 = __shfl_sync(0xffffffffu, y[2], s0), v2 = __shfl_sync(0xffffffffu, y[3], s0);
                const float u3 = __shfl_sync(0xffffffffu, y[2], s1), v3 = __shfl_sync(0xffffffffu, y[3], s1);
                yb[0] = odd ? v0 : u0; yb[1] = odd ? v1 : u1; yb[2] = odd ? v2 : u2; yb[3] = odd ? v3 : u3;
              }
              float oacc[2][4];
#pragma unroll
              for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < 4; ++i) oacc[u][i] = 0.f;
              const float* ta = Tf + (16 * a + g) * LDT + 16 * a + t4;
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                const float af[4] = {-ta[8 * ks], -ta[8 * LDT + 8 * ks], -ta[8 * ks + 4], -ta[8 * LDT + 8 * ks + 4]};
                const float bf[2] = {yb[2 * ks], yb[2 * ks + 1]};
                mma_1xtf32(oacc[ks], af, bf);
              }
              float o4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) o4[i] = oacc[0][i] + oacc[1][i];
              float* to = Tf + (16 * a + g) * LDT + 16 * b + n0 + 2 * t4;
              *reinterpret_cast<float2*>(to) = make_float2(o4[0], o4[1]);
              *reinterpret_cast<float2*>(to + 8 * LDT) = make_float2(o4[2], o4[3]);
            } else if (d == 1) {  // warps 6-7: rows 0-15 (items 0-127)
              pack_tp(tid - 192);
              pack_tp(tid - 192 + 64);
            } else if (d == 2) {  // warps 4-7: rows 16-31 (items 128-255)
              pack_tp(tid);
            } else {  // warps 2-7: rows 32-47 (items 256-383), one per thread of warps 2-5
              if (tid < 192) pack_tp(tid + 192);
            }
            sync_wg();
          }
        }
        if (tid < 128) pack_tp(384 + tid);  // rows 48-63
      }
      // A partial last chunk: the v tile's rows t >= L hold the next sequence's tokens (or the
      // zero fill past the tensor).  T' has zero columns there (beta = 0), but 0 * Inf or NaN is
      // NaN, so the rows are cleared: a sequence must not see its neighbour's values at all.
      if (L < C) {
        if (!wg_wait(&m->full_v, par)) { ok = false; break; }
        for (int idx = tid; idx < (C - L) * 16; idx += kCompute) {
          const int t = L + (idx >> 4), c16 = idx & 15;  // a row's 16-byte chunks, either block
          at16(sm, OFF_V + (c16 >> 3) * 8192 + t * 128 + ((c16 & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      ops_arrive();  // ---------------------------------------------- UMMA: W = T' Kt, U' = T' V
      if (write_out && j > 0) epilogue_b(L_prev, tok_prev);  // in the shadow of the W|U' UMMAs
      if (!kOut) {  // pass 1: M's bf16 copy, column half wg of this warp's rows (the Gram is done)
        uint32_t v[64];
        tmem_ld32(tl + TM_M + 64 * wg, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tl + TM_M + 64 * wg + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
#pragma unroll
        for (int oc = 0; oc < 8; ++oc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]);
          at16(sm, (wg ? OFF_MC1 : OFF_MC0) + sw128_oct(row, oc, 16384)) = pack8(f);
        }
      }
      {
        const bool r = wg_wait(&m->mma, mph & 1u);
        ++mph;
        tc_fence_after();
        if (!r) { ok = false; break; }
      }
      if (tid == 0) {  // v and the k rows (e^{gamma} k in place) consumed
        mbar_arrive(&m->empty_v);
        mbar_arrive(&m->empty_k);
        if (stage_gate && j > 0) mbar_arrive(&m->empty_gate);  // chunk j - 1's epilogue is done
      }

      // ---------------------------------------------------------------- -W -> bf16
      // lane l < 16: row 16 q + l, columns 32 wg ..; lane l + 16: the same row, columns 64 + 32 wg ..
      {
        const int t = 16 * q4 + (lane & 15);
        const int c0 = (lane >> 4) * 64 + wg * 32;
        uint32_t v[32];
        tmem_ld32(tl + tm_wu + 32 * wg, v);
        tmem_wait_ld();
#pragma unroll
        for (int oc = 0; oc < 4; ++oc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = -__uint_as_float(v[8 * oc + e]);
          at16(sm, OFF_KL + sw128_oct(t, (c0 >> 3) + oc, 8192)) = pack8(f);
        }
      }
      ops_arrive();  // ---------------------------------------------- UMMA: U = U' - W S0 ; O = Qt S0
      // in the shadow of these UMMAs (they read the bf16 copy of S, not TMEM columns [0,128)):
      // S <- Diag(e^{gamma_C}) S in TMEM, then the next chunk's decay scan, whose g tile the
      // producer fetched during this chunk; its release lets the producer fetch the one after
      {
        const float ec = m->ec[row];
#pragma unroll
        for (int hb = 0; hb < (kOut ? 2 : 4); ++hb) {  // (pass 1: the rows of M too)
          const uint32_t c0 = (hb < 2 ? TM_S : TM_M) + 64 * wg + 32 * (hb & 1);
          uint32_t v[32];
          tmem_ld32(tl + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __float_as_uint(__uint_as_float(v[jj]) * ec);
          tmem_st32(tl + c0, v);
        }
        tmem_wait_st();
      }
      bool next_ok = true;
      if (j + 1 < nchunks) {
        next_ok = wg_wait(&m->full_g, par ^ 1u);
        if (next_ok) {
          scan(min(C, seg.len - (j + 1) * C), gl);
          if (tid == 0) mbar_arrive(&m->empty_g);
        }
      }
      {
        const bool r = wg_wait(&m->mma, mph & 1u);
        ++mph;
        tc_fence_after();
        if (!r || !next_ok) { ok = false; break; }
      }
      if (tid == 0 && write_out) mbar_arrive(&m->empty_q);  // the q rows (e^{gamma} q in place) consumed

      // ---------------------------------------------------------------- U -> bf16 (same lane split as -W)
      {
        const int t = 16 * q4 + (lane & 15);
        const int c0 = (lane >> 4) * 64 + wg * 32;
        uint32_t v[32];
        tmem_ld32(tl + tm_wu + 64 + 32 * wg, v);
        tmem_wait_ld();
#pragma unroll
        for (int oc = 0; oc < 4; ++oc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]);
          at16(sm, OFF_KL + sw128_oct(t, (c0 >> 3) + oc, 8192)) = pack8(f);
        }
        if (!kOut) {  // pass 1: U_M over T' and P (the W|U' UMMAs that read T' are done)
          tmem_ld32(tl + TM_UM + 32 * wg, v);
          tmem_wait_ld();
#pragma unroll
          for (int oc = 0; oc < 4; ++oc) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * oc + e]);
            at16(sm, OFF_UM + sw128_oct(t, (c0 >> 3) + oc, 8192)) = pack8(f);
          }
        }
      }
      ops_arrive();  // ---------------------------------------------- UMMA: O += P U ; S += Kh^T U
      {
        const bool r = wg_wait(&m->mma, mph & 1u);
        ++mph;
        tc_fence_after();
        if (!r) { ok = false; break; }
      }

      L_prev = L;
      tok_prev = tok;
    }
    if (ok && write_out && nchunks > 0) {
      ok = !stage_gate || wg_wait(&m->full_gate, (uint32_t)((nchunks - 1) & 1));
      if (ok) {
        epilogue_a(L_prev, tok_prev);
        epilogue_b(L_prev, tok_prev);
      }
    }

    // ---------------------------------------------------------------- end state
    if (ok) {
      float* dst = nullptr;
      if (kOut && seg.last && p.final_state) dst = p.final_state + ((size_t)seg.seq * H + h) * unit_state;
      size_t ld = DV;
      if (!kOut) {  // pass 1: the (S_loc | M) block of the slot, row stride dv + dk
        ld = DV + DK;
        dst = p.ws_local + ((size_t)seg.slot * H + h) * (size_t)DK * ld;
      }
      float* sdst = kOut && nchunks > 0 ? snap_dst(seg.len) : nullptr;  // a snapshot boundary at the segment end
      if (dst || sdst) {
#pragma unroll
        for (int hb = 0; hb < (kOut ? 2 : 4); ++hb) {
          const int c0 = wg * 64 + (hb & 1) * 32;  // column of S (hb < 2) or of M
          uint32_t v[32];
          tmem_ld32(tl + (hb < 2 ? TM_S : TM_M) + c0, v);
          tmem_wait_ld();
          const int cd = (hb < 2 ? 0 : DV) + c0;
#pragma unroll
          for (int jj = 0; jj < 32; jj += 4) {
            const float4 x = make_float4(__uint_as_float(v[jj]), __uint_as_float(v[jj + 1]),
                                         __uint_as_float(v[jj + 2]), __uint_as_float(v[jj + 3]));
            if (dst) *reinterpret_cast<float4*>(dst + (size_t)row * ld + cd + jj) = x;
            if (sdst && hb < 2) *reinterpret_cast<float4*>(sdst + (size_t)row * DV + c0 + jj) = x;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The body is compiled twice: with outputs, and without them for the split's pass-1 roles
// (no q, no P, no Q.S or P.U chains, no epilogue). A CTA's role is uniform, so each CTA runs one
// copy, and the output copy carries no run-time tests of the role.
template <bool kPre>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ Plan plan, const __grid_constant__ TcMaps maps, const ChunkParams p) {
  const int role = plan.seg[blockIdx.x / plan.H].role;
  if (role == kRoleWhole || role == kRoleFromWs)
    chunk_tc_body<kPre, true>(plan, maps, p);
  else
    chunk_tc_body<kPre, false>(plan, maps, p);
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
      !make_map(&maps.v, p.v, p.H, T) || (p.gate && !make_map(&maps.gate, p.gate, p.H, T)))
    return cudaErrorInvalidValue;
  const bool pre = (p.flags & (KDA_FLAG_G_LOGITS | KDA_FLAG_QK_L2NORM)) != 0;
  auto kern = pre ? chunk_tc_kernel<true> : chunk_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<plan.n_seg * plan.H, kThreads, SMEM_BYTES, stream>>>(plan, maps, p);
  return cudaGetLastError();
}

}  // namespace kda
