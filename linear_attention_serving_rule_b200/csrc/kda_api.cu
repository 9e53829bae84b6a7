// kda_api.cu -- the C ABI of libkda: argument validation, work planning and dispatch.
//
// Host-side only (no kernels here).  Every check that can fail on the host runs before
// the first CUDA call, so a rejected call has no side effect on the device.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "kda_internal.cuh"

namespace kda {
namespace {

// Number of SMs the automatic sequence split plans for (B200: 148).  A constant, so that
// kda_chunk_fwd_workspace_size and kda_chunk_fwd agree without querying a device.
constexpr int kPlanSMs = 148;
constexpr int kSegAlign = 64;     // segment lengths are multiples of the largest chunk
constexpr int kMinAutoSeg = 2048; // automatic split: tokens per segment at least this
constexpr size_t kErrBytes = 256;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
// beta is read with scalar loads: element alignment is enough.
bool aligned_elem(const void* p, kda_dtype dt) { return ((uintptr_t)p & (dt == KDA_BF16 ? 1u : 3u)) == 0; }

struct SeqSpan {
  int32_t tok0, len, seq;
};

struct Layout {
  std::vector<SeqSpan> seqs;   // every sequence
  std::vector<int32_t> nseg;   // segments per sequence (1 = not split)
  std::vector<int32_t> seglen; // segment length per sequence
  std::vector<int32_t> slot0;  // first workspace slot of a split sequence
  int32_t slots = 0;
  bool any_split = false;
};

kda_status validate(const kda_chunk_args* a) {
  if (!a) return KDA_ERR_INVALID_ARGUMENT;
  if (a->num_seqs < 0 || a->total_tokens < 0 || a->H <= 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->total_tokens > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (a->dtype != KDA_BF16 && a->dtype != KDA_F32) return KDA_ERR_INVALID_ARGUMENT;
  if (a->dk <= 0 || a->dv <= 0) return KDA_ERR_INVALID_ARGUMENT;
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128)) return KDA_ERR_UNSUPPORTED;
  if (a->split_segments < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (!(a->eps >= 0.f) || !(a->scale >= 0.f)) return KDA_ERR_INVALID_ARGUMENT;
  if (a->num_seqs == 0 && a->total_tokens != 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->total_tokens > 0) {
    const void* req[] = {a->q, a->k, a->v, a->g, a->out};
    for (const void* p : req)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    if (!a->beta || !aligned_elem(a->beta, a->dtype)) return KDA_ERR_INVALID_ARGUMENT;
    if (a->gate && !aligned16(a->gate)) return KDA_ERR_INVALID_ARGUMENT;
  }
  if (a->norm_weight && !aligned16(a->norm_weight)) return KDA_ERR_INVALID_ARGUMENT;
  if (a->initial_state && !aligned16(a->initial_state)) return KDA_ERR_INVALID_ARGUMENT;
  if (a->final_state && !aligned16(a->final_state)) return KDA_ERR_INVALID_ARGUMENT;
  if (a->snapshots) {
    if (!aligned16(a->snapshots)) return KDA_ERR_INVALID_ARGUMENT;
    if (a->snapshot_interval <= 0 || a->snapshot_interval % 64 != 0) return KDA_ERR_INVALID_ARGUMENT;
  }
  if (a->cu_seqlens) {
    if (a->cu_seqlens[0] != 0) return KDA_ERR_INVALID_ARGUMENT;
    for (int32_t n = 0; n < a->num_seqs; ++n)
      if (a->cu_seqlens[n + 1] < a->cu_seqlens[n]) return KDA_ERR_INVALID_ARGUMENT;
    if ((int64_t)a->cu_seqlens[a->num_seqs] != a->total_tokens) return KDA_ERR_INVALID_ARGUMENT;
  } else if (a->num_seqs > 0 && a->total_tokens % a->num_seqs != 0) {
    return KDA_ERR_INVALID_ARGUMENT;
  }
  return KDA_OK;
}

int32_t round_up(int64_t x, int32_t m) { return (int32_t)(((x + m - 1) / m) * m); }

// bf16 with dk = dv = 128 runs on the tensor cores; everything else (and the unbounded-decay
// path) on the fp32 CUDA-core kernel.
bool uses_tensor_cores(const kda_chunk_args* a) {
  return a->dtype == KDA_BF16 && a->dk == 128 && a->dv == 128 &&
         !(a->flags & (KDA_FLAG_FORCE_SIMT | KDA_FLAG_UNBOUNDED_DECAY));
}

int64_t waves(int64_t units) { return (units + kPlanSMs - 1) / kPlanSMs; }

// Automatic segment count for `busy` (sequence, head) units whose longest sequence has `chunks`
// 64-token chunks: the split runs launch A (pass 1 of every segment but the last: one unit on the
// augmented state [S_loc | M] each), the combine, and launch B (every segment from its start
// state, with outputs).  In chunk times of one unit, a launch takes its waves times the chunks of
// a segment, and the combine about kCombineStep per segment boundary it chains (one dk x dk by
// dk x dv product per (sequence, head) in fp32: measured ~37 us against ~9 us per chunk).  The P
// with the least time is taken, if it saves at least a fifth of the unsplit time.
constexpr int64_t kCombineStep = 4;
int32_t auto_segments(int64_t busy, int64_t chunks) {
  int32_t best = 1;
  double best_t = 0.8 * (double)chunks;
  for (int32_t P = 2; P <= 64; ++P) {
    const int64_t seg_chunks = (chunks + P - 1) / P;
    const double t = (double)((waves(busy * (int64_t)(P - 1)) + waves(busy * (int64_t)P)) * seg_chunks +
                              kCombineStep * (P - 1));
    if (t < best_t - 1e-9) {
      best_t = t;
      best = P;
    }
  }
  return best;
}

Layout make_layout(const kda_chunk_args* a) {
  Layout L;
  const int32_t N = a->num_seqs;
  L.seqs.resize(N);
  for (int32_t n = 0; n < N; ++n) {
    int32_t t0, len;
    if (a->cu_seqlens) {
      t0 = a->cu_seqlens[n];
      len = a->cu_seqlens[n + 1] - a->cu_seqlens[n];
    } else {
      len = (int32_t)(a->total_tokens / N);
      t0 = n * len;
    }
    L.seqs[n] = {t0, len, n};
  }
  // Sequence split: automatic when the (sequence, head) units cannot fill half the GPU.
  int64_t busy = 0, max_len = 0;
  for (const auto& s : L.seqs) {
    busy += (s.len > 0) ? a->H : 0;
    max_len = std::max<int64_t>(max_len, s.len);
  }
  int32_t P = 1;
  bool auto_mode = a->split_segments == 0;
  if (auto_mode) {
    if (busy > 0 && busy * 2 <= kPlanSMs) P = auto_segments(busy, (max_len + 63) / 64);
  } else {
    P = a->split_segments;
  }
  L.nseg.assign(N, 1);
  L.seglen.assign(N, 0);
  L.slot0.assign(N, -1);
  for (int32_t n = 0; n < N; ++n) {
    const int32_t len = L.seqs[n].len;
    L.seglen[n] = len;
    if (P <= 1 || len <= kSegAlign) continue;
    int32_t p = P;
    if (auto_mode) p = (int32_t)std::min<int64_t>(p, len / kMinAutoSeg);
    if (p <= 1) continue;
    const int32_t sl = round_up((len + p - 1) / p, kSegAlign);
    const int32_t np = (len + sl - 1) / sl;
    if (np <= 1) continue;
    L.nseg[n] = np;
    L.seglen[n] = sl;
    L.slot0[n] = L.slots;
    L.slots += np;
    L.any_split = true;
  }
  return L;
}

size_t workspace_bytes(const kda_chunk_args* a, const Layout& L) {
  size_t b = kErrBytes;
  if (L.slots > 0) {
    const size_t per = (size_t)a->dk * a->dv + (size_t)a->dk * (a->dv + a->dk);
    b += (size_t)L.slots * a->H * per * sizeof(float);
  }
  return b;
}

Seg make_seg(int32_t t0, int32_t len, int32_t seq, int32_t role, int32_t slot, int32_t last) {
  return Seg{t0, len, seq, role, slot, last, -1, 0};
}

// Snapshot rows: sequence n's snapshots start at row base[n] = sum_{m<n} floor(len_m / I).
std::vector<int64_t> snapshot_bases(const Layout& L, int32_t I, int64_t* total) {
  std::vector<int64_t> base(L.seqs.size());
  int64_t acc = 0;
  for (size_t n = 0; n < L.seqs.size(); ++n) {
    base[n] = acc;
    acc += L.seqs[n].len / I;
  }
  if (total) *total = acc;
  return base;
}

// The first snapshot boundary inside a segment that starts q0 tokens into its sequence: the
// smallest multiple of I above q0, if the segment reaches it.
void assign_snapshot(Seg& s, int32_t q0, int32_t I, int64_t base) {
  const int64_t p1 = ((int64_t)q0 / I + 1) * I;
  const int64_t off = p1 - q0;
  if (off <= s.len) {
    s.snap = (int32_t)(base + p1 / I - 1);
    s.snap_off = (int32_t)off;
  }
}

// Launch `segs` (all of one role class) in batches of kPlanMax, longest first.
cudaError_t run_segments(std::vector<Seg>& segs, const ChunkParams& p, kda_dtype dtype, bool use_tc,
                         cudaStream_t stream) {
  std::stable_sort(segs.begin(), segs.end(), [](const Seg& x, const Seg& y) { return x.len > y.len; });
  static thread_local Plan plan;  // 30 KB: kept off the stack
  for (size_t b = 0; b < segs.size(); b += kPlanMax) {
    const size_t n = std::min<size_t>(kPlanMax, segs.size() - b);
    plan.n_seg = (int32_t)n;
    plan.H = p.H;
    for (size_t i = 0; i < n; ++i) plan.seg[i] = segs[b + i];
    cudaError_t e = use_tc ? launch_chunk_tc(plan, p, stream) : launch_chunk_simt(plan, p, dtype, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" kda_status kda_chunk_fwd_snapshot_count(const kda_chunk_args* a, int64_t* n_snap) {
  // reads the sequence layout and the interval only
  if (!a || !n_snap) return KDA_ERR_INVALID_ARGUMENT;
  if (a->num_seqs < 0 || a->total_tokens < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->num_seqs == 0 && a->total_tokens != 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->snapshot_interval <= 0 || a->snapshot_interval % 64 != 0) return KDA_ERR_INVALID_ARGUMENT;
  int64_t n = 0;
  for (int32_t i = 0; i < a->num_seqs; ++i) {
    int64_t len;
    if (a->cu_seqlens) {
      if (a->cu_seqlens[i + 1] < a->cu_seqlens[i]) return KDA_ERR_INVALID_ARGUMENT;
      len = a->cu_seqlens[i + 1] - a->cu_seqlens[i];
    } else {
      if (a->total_tokens % a->num_seqs != 0) return KDA_ERR_INVALID_ARGUMENT;
      len = a->total_tokens / a->num_seqs;
    }
    n += len / a->snapshot_interval;
  }
  if (a->cu_seqlens && (a->cu_seqlens[0] != 0 || (int64_t)a->cu_seqlens[a->num_seqs] != a->total_tokens))
    return KDA_ERR_INVALID_ARGUMENT;
  *n_snap = n;
  return KDA_OK;
}

extern "C" kda_status kda_chunk_fwd_workspace_size(const kda_chunk_args* a, size_t* bytes) {
  if (!bytes) return KDA_ERR_INVALID_ARGUMENT;
  kda_status s = validate(a);
  if (s != KDA_OK) return s;
  *bytes = workspace_bytes(a, make_layout(a));
  return KDA_OK;
}

extern "C" kda_status kda_chunk_fwd(const kda_chunk_args* a, void* cuda_stream) {
  kda_status s = validate(a);
  if (s != KDA_OK) return s;
  const Layout L = make_layout(a);
  if (!a->workspace || ((uintptr_t)a->workspace & 255u) != 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->workspace_bytes < workspace_bytes(a, L)) return KDA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = (cudaStream_t)cuda_stream;

  ChunkParams p;
  p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta; p.gate = a->gate;
  p.norm_weight = a->norm_weight;
  p.initial_state = a->initial_state;
  p.out = a->out;
  p.final_state = a->final_state;
  p.error_word = (uint32_t*)a->workspace;
  p.snapshots = a->snapshots;
  p.snap_interval = a->snapshots ? a->snapshot_interval : 0;
  float* ws = (float*)((char*)a->workspace + kErrBytes);
  p.ws_state = L.slots ? ws : nullptr;
  p.ws_local = L.slots ? ws + (size_t)L.slots * a->H * a->dk * a->dv : nullptr;
  p.total_tokens = a->total_tokens;
  p.H = a->H; p.dk = a->dk; p.dv = a->dv;
  p.scale = a->scale > 0.f ? a->scale : 1.0f / sqrtf((float)a->dk);
  p.eps = a->eps;
  p.flags = a->flags;

  if (cudaMemsetAsync(a->workspace, 0, sizeof(uint32_t), stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (a->num_seqs == 0) return KDA_OK;

  const bool use_tc = uses_tensor_cores(a);

  // Launch A: pass 1 of every segment of a split sequence but the last (local state from zero and
  // the transition matrix, one unit on the augmented state each).  Then the combine, which chains
  // the start states from the initial state.  Then launch B: every segment of the split sequences
  // from its start state, and every unsplit sequence from its initial state (outputs, snapshots,
  // final states).  Each launch runs one kind of unit only: on the tensor cores a launch that
  // mixed the pass-1 body with the output body measured some of its CTAs 1.7x slower than either
  // kind alone.
  std::vector<Seg> local, rest;
  std::vector<int64_t> snap_base;
  if (a->snapshots) snap_base = snapshot_bases(L, a->snapshot_interval, nullptr);
  // segments that carry the true state write the snapshots inside them
  auto with_snap = [&](Seg sg, int32_t n) {
    if (a->snapshots) assign_snapshot(sg, sg.tok0 - L.seqs[n].tok0, a->snapshot_interval, snap_base[n]);
    return sg;
  };
  for (int32_t n = 0; n < a->num_seqs; ++n) {
    const SeqSpan& sp = L.seqs[n];
    const int32_t np = L.nseg[n];
    if (np == 1) {
      rest.push_back(with_snap(make_seg(sp.tok0, sp.len, sp.seq, kRoleWhole, -1, 1), n));
      continue;
    }
    const int32_t sl = L.seglen[n], b = L.slot0[n];
    for (int32_t q = 0; q < np; ++q) {
      const int32_t t0 = sp.tok0 + q * sl;
      const int32_t len = std::min(sl, sp.len - q * sl);
      if (q < np - 1) local.push_back(make_seg(t0, len, sp.seq, kRoleLocal, b + q, 0));
      rest.push_back(with_snap(make_seg(t0, len, sp.seq, kRoleFromWs, b + q, q == np - 1 ? 1 : 0), n));
    }
  }
  cudaError_t e = local.empty() ? cudaSuccess : run_segments(local, p, a->dtype, use_tc, stream);
  if (e == cudaSuccess && L.any_split) {
    // combine: S_start(0) = the initial state, S_start(q+1) = M_q S_start(q) + S_loc(q),
    // sequential over q per (sequence, head)
    static thread_local Plan plan;
    plan.H = a->H;
    plan.n_seg = 0;
    for (int32_t n = 0; n < a->num_seqs && e == cudaSuccess; ++n) {
      if (L.nseg[n] <= 1) continue;
      plan.seg[plan.n_seg++] = make_seg(L.seqs[n].tok0, L.nseg[n], L.seqs[n].seq, kRoleLocal, L.slot0[n], 0);
      if (plan.n_seg == kPlanMax) {
        e = launch_split_combine(plan, p, 0, stream);
        plan.n_seg = 0;
      }
    }
    if (e == cudaSuccess && plan.n_seg > 0) e = launch_split_combine(plan, p, 0, stream);
  }
  if (e == cudaSuccess && !rest.empty()) e = run_segments(rest, p, a->dtype, use_tc, stream);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status kda_decode_step(const kda_decode_args* a, void* cuda_stream) {
  if (!a) return KDA_ERR_INVALID_ARGUMENT;
  if (a->N < 0 || a->H <= 0 || a->num_slots < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (a->dtype != KDA_BF16 && a->dtype != KDA_F32) return KDA_ERR_INVALID_ARGUMENT;
  if (a->dk <= 0 || a->dv <= 0) return KDA_ERR_INVALID_ARGUMENT;
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128)) return KDA_ERR_UNSUPPORTED;
  if (!(a->eps >= 0.f) || !(a->scale >= 0.f)) return KDA_ERR_INVALID_ARGUMENT;
  if ((int64_t)a->N * a->H > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (a->tokens < 0) return KDA_ERR_INVALID_ARGUMENT;
  if ((int64_t)a->N * (a->tokens > 0 ? a->tokens : 1) * a->H > INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (a->position_states && !aligned16(a->position_states)) return KDA_ERR_INVALID_ARGUMENT;
  if (a->N > 0) {
    const void* req[] = {a->q, a->k, a->v, a->g, a->state, a->out};
    for (const void* p : req)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARGUMENT;
    if (!a->beta || !aligned_elem(a->beta, a->dtype)) return KDA_ERR_INVALID_ARGUMENT;
    if (a->gate && !aligned16(a->gate)) return KDA_ERR_INVALID_ARGUMENT;
    if (a->norm_weight && !aligned16(a->norm_weight)) return KDA_ERR_INVALID_ARGUMENT;
    if (!a->state_indices && a->num_slots < a->N) return KDA_ERR_INVALID_ARGUMENT;
    if (a->num_slots == 0) return KDA_ERR_INVALID_ARGUMENT;
  }
  if (a->N == 0) return KDA_OK;
  kda_decode_args b = *a;
  if (!(b.scale > 0.f)) b.scale = 1.0f / sqrtf((float)b.dk);
  return launch_decode(b, (cudaStream_t)cuda_stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status kda_read_device_error(const void* error_word, void* cuda_stream) {
  if (!error_word) return KDA_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize((cudaStream_t)cuda_stream) != cudaSuccess) return KDA_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, error_word, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
  if (w != 0 && cudaMemset((void*)error_word, 0, sizeof(w)) != cudaSuccess) return KDA_ERR_CUDA;
  return (kda_status)w;
}

extern "C" const char* kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARGUMENT: return "KDA_ERR_INVALID_ARGUMENT";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_WORKSPACE_TOO_SMALL: return "KDA_ERR_WORKSPACE_TOO_SMALL";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    case KDA_ERR_DECAY_OUT_OF_RANGE: return "KDA_ERR_DECAY_OUT_OF_RANGE";
    case KDA_ERR_BAD_STATE_INDEX: return "KDA_ERR_BAD_STATE_INDEX";
  }
  return "KDA_ERR_UNKNOWN";
}
