// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they run the layer:
// code being captured into a CUDA graph, or a runtime whose device memory pool is fixed when it
// starts.  For them the scratch that kda_chunk_fwd needs lives in a file-scope device array,
// created with the module on every GPU that loads this library and held until exit.  In host
// code the array's name is only a host-side handle, so its device address is looked up once per
// device (with that device current) and handed to kda_chunk_fwd as the workspace.
#include <mutex>

#include "kda_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_kda_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const kda_chunk_args* args, void* cuda_stream, const void** error_word) {
  if (!args) return KDA_ERR_INVALID_ARGUMENT;
  size_t need = 0;
  const kda_status s = kda_chunk_fwd_workspace_size(args, &need);
  if (s != KDA_OK) return s;
  if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_kda_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
      g_scratch_ptr[dev] = p;
    }
    ptr = g_scratch_ptr[dev];
  }
  kda_chunk_args a = *args;
  a.workspace = ptr;
  a.workspace_bytes = KDA_NOALLOC_SCRATCH_BYTES;
  if (error_word) *error_word = ptr;
  return kda_chunk_fwd(&a, cuda_stream);
}
