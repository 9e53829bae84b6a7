// kda_internal.cuh -- shared declarations of libkda's host API and its kernels.
//
// The work plan: a prefill call is cut into segments (a whole sequence, or a piece of
// one when a long sequence is split so that every SM has work).  A work unit is one
// (segment, head); units are launched longest segment first so that the block
// scheduler's in-order dispatch gives a longest-processing-time-first schedule.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

constexpr int kPlanMax = 960;  // segments per launch (the plan travels in the kernel parameters,
                               // which hold at most 32,764 bytes)

// Where a unit's start state comes from and where its end state goes.
enum SegRole : int32_t {
  kRoleWhole = 0,     // an unsplit sequence: start: initial_state (or 0); writes outputs;
                      //   end: final_state
  kRoleLocal = 1,     // split pass 1: start from [0 | I] (the augmented state [S | M], values
                      //   augmented by zeros), no outputs; end: workspace slot (S_loc | M)
  kRoleFromWs = 3,    // split pass 2: start from workspace start-state slot; writes outputs;
                      //   end state -> final_state if last segment of its sequence
};

struct Seg {
  int32_t tok0;   // first token (row of the packed [T_tot, H, d] tensors)
  int32_t len;    // tokens in the segment
  int32_t seq;    // sequence index (initial_state / final_state row)
  int32_t role;   // SegRole
  int32_t slot;   // workspace slot (split passes), -1 if unused
  int32_t last;   // 1 if this segment ends its sequence (writes final_state)
  int32_t snap;      // snapshot row of the first snapshot boundary inside the segment, -1 if none
  int32_t snap_off;  // that boundary's offset from the segment start, in tokens (1 .. len)
};

struct Plan {
  int32_t n_seg;
  int32_t H;
  Seg seg[kPlanMax];
};

// Common arguments of the prefill kernels (pointers already validated).
struct ChunkParams {
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
  float* ws_state;     // split: per-slot [dk, dv] start states (pass 2 reads), or null
  float* ws_local;     // split: per-slot [dk, dv + dk] (S_loc | M) from pass 1, or null
  uint32_t* error_word;
  float* snapshots;      // [n_snap, H, dk, dv] chunk-boundary states, or null
  int32_t snap_interval; // tokens between snapshot boundaries (a multiple of 64)
  int64_t total_tokens;  // rows of the packed tensors (tensor-map extent)
  int32_t H, dk, dv;
  float scale, eps;
  uint32_t flags;
};

// Device-side helpers: compiled by nvcc only, so that the host code of the C ABI also builds
// with a plain C++ compiler (the host-side sanitizer tests do that).
#ifdef __CUDACC__
// Set the device error word once (the first error wins).
__device__ __forceinline__ void report_error(uint32_t* word, kda_status s) {
  if (word) atomicCAS(word, 0u, (uint32_t)s);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
#endif  // __CUDACC__

// Launchers (host).  Each returns cudaSuccess or the launch error.
cudaError_t launch_decode(const kda_decode_args& a, cudaStream_t stream);
cudaError_t launch_chunk_simt(const Plan& plan, const ChunkParams& p, kda_dtype dtype, cudaStream_t stream);
cudaError_t launch_chunk_tc(const Plan& plan, const ChunkParams& p, cudaStream_t stream);
cudaError_t launch_split_combine(const Plan& plan, const ChunkParams& p, int32_t segs_per_seq,
                                 cudaStream_t stream);

}  // namespace kda
