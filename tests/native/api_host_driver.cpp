// api_host_driver.cpp -- runs the host side of libkda's C ABI (kda_api.cu: argument checks,
// the work plan, the sequence split, snapshot rows, workspace sizing) under AddressSanitizer and
// UndefinedBehaviorSanitizer, with no GPU.  The kernel launchers and the few CUDA runtime calls
// the host code makes are replaced by stubs that record what would have been launched, and the
// recorded plans are checked against invariants: the final pass tiles every sequence exactly,
// launches run their segments longest first, split segments are whole chunks, pass 1 and the
// combine cover the split sequences, snapshot rows follow the layout of include/kda.h.
// Test infrastructure: built and run by tests/test_host_sanitizers.py.
#include <stdio.h>
#include <stdlib.h>

#include <algorithm>
#include <map>
#include <vector>

#include "kda.h"
#include "kda_internal.cuh"

namespace {
struct Launch {
  char kind;  // 't' tensor-core chunk, 's' CUDA-core chunk, 'c' split combine, 'd' decode
  int H;
  std::vector<kda::Seg> segs;
};
std::vector<Launch> g_launches;
int g_fail_launch = -1;  // index of the launch that reports a failure, or -1

cudaError_t record(char kind, const kda::Plan* plan, int H) {
  Launch L{kind, H, {}};
  if (plan) L.segs.assign(plan->seg, plan->seg + plan->n_seg);
  g_launches.push_back(L);
  return (int)g_launches.size() - 1 == g_fail_launch ? cudaErrorLaunchFailure : cudaSuccess;
}
}  // namespace

namespace kda {
cudaError_t launch_decode(const kda_decode_args& a, cudaStream_t) { return record('d', nullptr, a.H); }
cudaError_t launch_chunk_simt(const Plan& plan, const ChunkParams&, kda_dtype, cudaStream_t) {
  return record('s', &plan, plan.H);
}
cudaError_t launch_chunk_tc(const Plan& plan, const ChunkParams&, cudaStream_t) { return record('t', &plan, plan.H); }
cudaError_t launch_split_combine(const Plan& plan, const ChunkParams&, int32_t, cudaStream_t) {
  return record('c', &plan, plan.H);
}
}  // namespace kda

extern "C" {
cudaError_t cudaMemsetAsync(void*, int, size_t, cudaStream_t) { return cudaSuccess; }
cudaError_t cudaStreamSynchronize(cudaStream_t) { return cudaSuccess; }
cudaError_t cudaMemcpy(void* dst, const void*, size_t n, cudaMemcpyKind) {
  for (size_t i = 0; i < n; ++i) static_cast<unsigned char*>(dst)[i] = 0;
  return cudaSuccess;
}
cudaError_t cudaMemset(void*, int, size_t) { return cudaSuccess; }
}

#define CHECK(c)                                                    \
  do {                                                              \
    if (!(c)) {                                                     \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      exit(1);                                                      \
    }                                                               \
  } while (0)

// fake device addresses: never dereferenced by host code, only checked for NULL and alignment
void* dev(uintptr_t i) { return reinterpret_cast<void*>((uintptr_t)0x7f0000000000ull + i * 0x100000ull); }

kda_chunk_args base_args(int32_t N, int64_t T, const int32_t* cu, int H) {
  kda_chunk_args a{};
  a.num_seqs = N;
  a.total_tokens = T;
  a.cu_seqlens = cu;
  a.H = H;
  a.dk = 128;
  a.dv = 128;
  a.dtype = KDA_BF16;
  a.q = dev(1); a.k = dev(2); a.v = dev(3); a.g = dev(4); a.beta = dev(5); a.gate = dev(6);
  a.out = dev(7);
  a.final_state = static_cast<float*>(dev(8));
  a.eps = 1e-6f;
  return a;
}

// Run kda_chunk_fwd with a big enough workspace and check the recorded plan.
void run_and_check(kda_chunk_args a, const std::vector<int32_t>& lens, bool expect_split) {
  size_t ws = 0;
  CHECK(kda_chunk_fwd_workspace_size(&a, &ws) == KDA_OK);
  CHECK(ws >= 256);
  a.workspace = dev(9);
  a.workspace_bytes = ws;
  g_launches.clear();
  CHECK(kda_chunk_fwd(&a, nullptr) == KDA_OK);
  const int N = (int)lens.size();
  std::vector<int64_t> tok0(N + 1, 0);
  for (int n = 0; n < N; ++n) tok0[n + 1] = tok0[n] + lens[n];
  std::map<int, std::vector<kda::Seg>> final_pass;
  bool any_split = false;
  int combine_units = 0;
  std::map<int, int> pass1;  // slot -> count of pass-1 results
  int stage = 0;  // 0: pass 1, 1: combine, 2: outputs; launches never go back a stage
  for (const Launch& L : g_launches) {
    CHECK(L.kind == 't' || L.kind == 's' || L.kind == 'c');
    CHECK(L.H == a.H);
    CHECK(!L.segs.empty() && (int)L.segs.size() <= kda::kPlanMax);
    if (L.kind == 'c') {
      CHECK(stage <= 1);
      stage = 1;
      for (const auto& s : L.segs) {
        CHECK(s.len >= 2 && s.slot >= 0);  // the segment count travels in len
        combine_units += 1;
      }
      continue;
    }
    for (size_t i = 1; i < L.segs.size(); ++i) CHECK(L.segs[i - 1].len >= L.segs[i].len);  // longest first
    // one kind of unit per launch: pass 1 only, or output units only
    const bool is_pass1 = L.segs[0].role == kda::kRoleLocal;
    for (const auto& s : L.segs) CHECK((s.role == kda::kRoleLocal) == is_pass1);
    CHECK(is_pass1 ? stage == 0 : true);
    if (!is_pass1) stage = 2;
    for (const auto& s : L.segs) {
      CHECK(s.seq >= 0 && s.seq < N);
      // an empty unit only for an empty sequence (it copies the initial state to the final one)
      CHECK(s.len > 0 || (lens[s.seq] == 0 && s.role == kda::kRoleWhole && s.last == 1));
      CHECK(s.tok0 >= tok0[s.seq] && s.tok0 + s.len <= tok0[s.seq + 1]);
      if (s.role == kda::kRoleWhole || s.role == kda::kRoleFromWs) {
        final_pass[s.seq].push_back(s);
      } else {
        any_split = true;
        CHECK(s.slot >= 0);
        CHECK((s.tok0 - tok0[s.seq]) % 64 == 0 && s.len % 64 == 0);  // pass 1 never holds a sequence's tail
        pass1[s.slot] += 1;
      }
    }
  }
  for (auto& kv : final_pass) any_split |= kv.second.size() > 1;
  CHECK(any_split == expect_split);
  for (int n = 0; n < N; ++n) {
    auto& v = final_pass[n];
    if (lens[n] == 0) {  // one empty unit, whose final state is its initial state
      CHECK(v.size() == 1 && v[0].len == 0 && v[0].tok0 == tok0[n]);
      continue;
    }
    std::sort(v.begin(), v.end(), [](const kda::Seg& x, const kda::Seg& y) { return x.tok0 < y.tok0; });
    int64_t at = tok0[n];
    for (size_t i = 0; i < v.size(); ++i) {
      CHECK(v[i].tok0 == at);
      at += v[i].len;
      CHECK(v[i].last == (i + 1 == v.size() ? 1 : 0));
      if (i + 1 < v.size()) CHECK(v[i].len % 64 == 0);
      // an unsplit sequence runs whole from its initial state; every segment of a split one from
      // the start state the combine left in its slot, and all but the last also ran pass 1
      CHECK(v[i].role == (v.size() == 1 ? kda::kRoleWhole : kda::kRoleFromWs));
      if (v.size() > 1) CHECK(pass1.count(v[i].slot) == (i + 1 < v.size() ? 1u : 0u));
    }
    CHECK(at == tok0[n + 1]);
  }
  for (const auto& kv : pass1) CHECK(kv.second == 1);
  CHECK(any_split == (combine_units > 0));  // a split sequence always needs its start states chained
}

int main() {
  // ---------------------------------------------------------------- argument checks
  const int32_t cu3[] = {0, 100, 100, 350};
  kda_chunk_args a = base_args(3, 350, cu3, 4);
  size_t ws = 0;
  CHECK(kda_chunk_fwd_workspace_size(&a, &ws) == KDA_OK);
  CHECK(kda_chunk_fwd_workspace_size(nullptr, &ws) == KDA_ERR_INVALID_ARGUMENT);
  CHECK(kda_chunk_fwd_workspace_size(&a, nullptr) == KDA_ERR_INVALID_ARGUMENT);
  {
    kda_chunk_args b = a; b.q = nullptr;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.k = static_cast<const char*>(a.k) + 8;  // misaligned
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.dk = 96;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_UNSUPPORTED);
    b = a; b.dk = -1;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    const int32_t bad[] = {0, 200, 100, 350};
    b = a; b.cu_seqlens = bad;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    const int32_t bad_end[] = {0, 100, 100, 349};
    b = a; b.cu_seqlens = bad_end;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.cu_seqlens = nullptr;  // 350 tokens do not split into 3 equal sequences
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.total_tokens = (int64_t)INT32_MAX + 1;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) != KDA_OK);
    b = a; b.eps = -1.f;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.split_segments = -2;
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.snapshots = static_cast<float*>(dev(10)); b.snapshot_interval = 100;  // not a multiple of 64
    CHECK(kda_chunk_fwd_workspace_size(&b, &ws) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.workspace = nullptr;
    CHECK(kda_chunk_fwd(&b, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    b = a; b.workspace = dev(9); b.workspace_bytes = 8;
    CHECK(kda_chunk_fwd(&b, nullptr) == KDA_ERR_WORKSPACE_TOO_SMALL);
    b = a; b.workspace = static_cast<char*>(dev(9)) + 16; b.workspace_bytes = 1 << 20;  // not 256-aligned
    CHECK(kda_chunk_fwd(&b, nullptr) == KDA_ERR_INVALID_ARGUMENT);
  }
  CHECK(g_launches.empty());  // nothing launched by a rejected call

  // ---------------------------------------------------------------- plans
  // dense B4 x T4096, H32: one tensor-core launch of four whole sequences, no split
  {
    kda_chunk_args b = base_args(4, 4 * 4096, nullptr, 32);
    run_and_check(b, {4096, 4096, 4096, 4096}, false);
    CHECK(g_launches.size() == 1 && g_launches[0].kind == 't' && g_launches[0].segs.size() == 4);
    size_t w = 0;
    CHECK(kda_chunk_fwd_workspace_size(&b, &w) == KDA_OK && w == 256);
  }
  // 64 ragged sequences (lengths from a fixed LCG in [128, 8192]), with a zero-length one
  {
    std::vector<int32_t> lens(64);
    uint32_t x = 12345;
    for (auto& l : lens) { x = x * 1664525u + 1013904223u; l = 128 + (int32_t)((x >> 8) % 8065); }
    lens[17] = 0;
    std::vector<int32_t> cu(65, 0);
    for (int i = 0; i < 64; ++i) cu[i + 1] = cu[i] + lens[i];
    kda_chunk_args b = base_args(64, cu[64], cu.data(), 32);
    run_and_check(b, lens, false);
    b.dtype = KDA_F32;  // the fp32 workload runs on the CUDA-core kernel
    run_and_check(b, lens, false);
    CHECK(g_launches[0].kind == 's');
  }
  // one 2^20-token sequence with 16 heads: the automatic split fills the GPU
  {
    const int32_t T = 1 << 20;
    const int32_t cu1[] = {0, T};
    kda_chunk_args b = base_args(1, T, cu1, 16);
    run_and_check(b, {T}, true);
    bool has_combine = false;
    for (const auto& L : g_launches) has_combine |= L.kind == 'c';
    CHECK(has_combine);
    size_t w = 0;
    CHECK(kda_chunk_fwd_workspace_size(&b, &w) == KDA_OK && w > 256);
  }
  // forced splits of ragged sequences (short ones stay whole), tensor-core and CUDA-core paths
  for (int split : {2, 3, 5, 64}) {
    const std::vector<int32_t> lens = {700, 64, 0, 1100, 130, 1};
    std::vector<int32_t> cu(lens.size() + 1, 0);
    for (size_t i = 0; i < lens.size(); ++i) cu[i + 1] = cu[i] + lens[i];
    kda_chunk_args b = base_args((int32_t)lens.size(), cu.back(), cu.data(), 3);
    b.split_segments = split;
    run_and_check(b, lens, true);
    b.flags = KDA_FLAG_FORCE_SIMT;
    run_and_check(b, lens, true);
  }
  // a failed launch is reported as KDA_ERR_CUDA and stops the call
  {
    const int32_t cu1[] = {0, 5000};
    kda_chunk_args b = base_args(1, 5000, cu1, 2);
    b.split_segments = 3;
    size_t w = 0;
    CHECK(kda_chunk_fwd_workspace_size(&b, &w) == KDA_OK);
    b.workspace = dev(9);
    b.workspace_bytes = w;
    g_launches.clear();
    g_fail_launch = 0;
    CHECK(kda_chunk_fwd(&b, nullptr) == KDA_ERR_CUDA);
    CHECK(g_launches.size() == 1);
    g_fail_launch = -1;
  }

  // ---------------------------------------------------------------- snapshot rows
  {
    const std::vector<int32_t> lens = {300, 0, 1024, 130, 2000};
    std::vector<int32_t> cu(lens.size() + 1, 0);
    for (size_t i = 0; i < lens.size(); ++i) cu[i + 1] = cu[i] + lens[i];
    const int32_t I = 128;
    for (int split : {1, 4}) {
      kda_chunk_args b = base_args((int32_t)lens.size(), cu.back(), cu.data(), 2);
      b.snapshots = static_cast<float*>(dev(11));
      b.snapshot_interval = I;
      b.split_segments = split;
      int64_t n_snap = -1;
      CHECK(kda_chunk_fwd_snapshot_count(&b, &n_snap) == KDA_OK);
      int64_t expect = 0;
      for (int32_t l : lens) expect += l / I;
      CHECK(n_snap == expect);
      run_and_check(b, lens, split > 1);
      // every snapshot row is assigned once, to the segment holding its boundary
      std::vector<int> seen(n_snap, 0);
      std::vector<int64_t> base(lens.size() + 1, 0);
      for (size_t n = 0; n < lens.size(); ++n) base[n + 1] = base[n] + lens[n] / I;
      for (const auto& L : g_launches) {
        if (L.kind == 'c') continue;
        for (const auto& s : L.segs) {
          if (s.role != kda::kRoleWhole && s.role != kda::kRoleFromWs) {
            CHECK(s.snap < 0);  // pass 1 does not carry the true state
            continue;
          }
          if (s.snap < 0) continue;
          const int64_t q0 = s.tok0 - cu[s.seq];
          const int64_t p = q0 + s.snap_off;
          CHECK(p % I == 0 && p > q0 && p <= q0 + s.len && p - I <= q0);
          CHECK(s.snap == base[s.seq] + p / I - 1);
          for (int64_t r = s.snap, pp = p; pp <= q0 + s.len; ++r, pp += I) seen[r] += 1;
        }
      }
      for (int64_t r = 0; r < n_snap; ++r) CHECK(seen[r] == 1);
    }
    kda_chunk_args b = base_args((int32_t)lens.size(), cu.back(), cu.data(), 2);
    b.snapshot_interval = 96;
    int64_t n_snap = 0;
    CHECK(kda_chunk_fwd_snapshot_count(&b, &n_snap) == KDA_ERR_INVALID_ARGUMENT);
  }

  // ---------------------------------------------------------------- decode
  {
    kda_decode_args d{};
    d.N = 4; d.H = 2; d.dk = 128; d.dv = 128; d.dtype = KDA_BF16;
    d.q = dev(1); d.k = dev(2); d.v = dev(3); d.g = dev(4); d.beta = dev(5); d.gate = dev(6);
    d.state = static_cast<float*>(dev(7)); d.num_slots = 4; d.out = dev(8); d.eps = 1e-6f;
    g_launches.clear();
    CHECK(kda_decode_step(&d, nullptr) == KDA_OK && g_launches.size() == 1);
    kda_decode_args e = d; e.num_slots = 3;  // identity map needs N slots
    CHECK(kda_decode_step(&e, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    e = d; e.state_indices = static_cast<const int32_t*>(dev(12)); e.num_slots = 1;
    CHECK(kda_decode_step(&e, nullptr) == KDA_OK);
    e = d; e.dv = 32;
    CHECK(kda_decode_step(&e, nullptr) == KDA_ERR_UNSUPPORTED);
    e = d; e.tokens = -1;
    CHECK(kda_decode_step(&e, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    e = d; e.position_states = reinterpret_cast<float*>(static_cast<char*>(dev(13)) + 4);
    CHECK(kda_decode_step(&e, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    e = d; e.v = nullptr;
    CHECK(kda_decode_step(&e, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    e = d; e.N = 0; e.q = nullptr;
    CHECK(kda_decode_step(&e, nullptr) == KDA_OK);
    CHECK(kda_read_device_error(nullptr, nullptr) == KDA_ERR_INVALID_ARGUMENT);
    CHECK(kda_read_device_error(dev(1), nullptr) == KDA_OK);
  }
  for (int s = 0; s <= 8; ++s) CHECK(kda_status_string((kda_status)s) != nullptr);
  printf("api host driver ok\n");
  return 0;
}
