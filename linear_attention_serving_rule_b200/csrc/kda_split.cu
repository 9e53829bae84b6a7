// kda_split.cu -- combine step of the intra-GPU sequence split.
//
// A long sequence (1M-token context: "Kimi K3 Architecture Explained", section
// "Architecture at a glance") with few heads leaves most SMs idle when each
// (sequence, head) is one serial unit.  The split cuts the sequence into segments.
// The recurrence is linear in its start state, so segment q maps its start state as
//
//     S_end(q) = M_q S_start(q) + S_loc(q)
//
// where pass 1 computed (S_loc(q) | M_q) by running the segment from [0 | I] with values
// augmented by zeros.  This kernel chains the segments from the sequence's initial state:
//
//     S_start(0) = S_init (zero without one),   S_start(q+1) = M_q S_start(q) + S_loc(q),
//     q = 0 .. nseg-2,
//
// and leaves every S_start(q) in the workspace for the pass that writes the outputs.
// Value columns are independent, so each CTA owns a block of 16 state columns of one
// (sequence, head) and walks the segments in order.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kCols = 16;
constexpr int kThreads = 256;

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) combine_kernel(const __grid_constant__ Plan plan,
                                                           const ChunkParams p) {
  __shared__ float sc[DK][kCols];
  const int H = plan.H;
  const Seg s = plan.seg[blockIdx.x / H];
  const int h = blockIdx.x % H;
  const int j0 = blockIdx.y * kCols;
  const int nseg = s.len;  // the plan carries the segment count in `len`
  const int b = s.slot;
  constexpr int LD = DV + DK;
  const int j = threadIdx.x % kCols;
  const int i0 = threadIdx.x / kCols;
  constexpr int RS = kThreads / kCols;  // row stride
  constexpr int NR = DK / RS;           // rows per thread

  const size_t unit = (size_t)DK * DV;
  const float* init = p.initial_state ? p.initial_state + ((size_t)s.seq * H + h) * unit : nullptr;
  float* st = p.ws_state + ((size_t)b * H + h) * unit;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const size_t e = (size_t)(i0 + RS * r) * DV + j0 + j;
    const float x = init ? init[e] : 0.f;
    sc[i0 + RS * r][j] = x;
    st[e] = x;
  }
  __syncthreads();
  for (int q = 0; q <= nseg - 2; ++q) {
    const float* loc = p.ws_local + ((size_t)(b + q) * H + h) * (size_t)DK * LD;
    float acc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int i = i0 + RS * r;
      const float* mrow = loc + (size_t)i * LD + DV;
      float a = loc[(size_t)i * LD + j0 + j];
      for (int m = 0; m < DK; ++m) a += mrow[m] * sc[m][j];
      acc[r] = a;
    }
    __syncthreads();
    float* nxt = p.ws_state + ((size_t)(b + q + 1) * H + h) * unit;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int i = i0 + RS * r;
      sc[i][j] = acc[r];
      nxt[(size_t)i * DV + j0 + j] = acc[r];
    }
    __syncthreads();
  }
}

template <int DK, int DV>
cudaError_t launch_t(const Plan& plan, const ChunkParams& p, cudaStream_t stream) {
  dim3 grid(plan.n_seg * plan.H, DV / kCols);
  combine_kernel<DK, DV><<<grid, kThreads, 0, stream>>>(plan, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_split_combine(const Plan& plan, const ChunkParams& p, int32_t, cudaStream_t stream) {
  if (plan.n_seg == 0) return cudaSuccess;
  if (p.dk == 128 && p.dv == 128) return launch_t<128, 128>(plan, p, stream);
  if (p.dk == 128 && p.dv == 64) return launch_t<128, 64>(plan, p, stream);
  if (p.dk == 64 && p.dv == 128) return launch_t<64, 128>(plan, p, stream);
  return launch_t<64, 64>(plan, p, stream);
}

}  // namespace kda
