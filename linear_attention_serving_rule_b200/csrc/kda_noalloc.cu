// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they run the layer:
// code being captured into a CUDA graph, or a runtime whose device memory pool is fixed when it
// starts.  For them the scratch that kda_chunk_fwd needs lives in a file-scope device array,
// created with the module on every GPU that loads this library and held until exit.  In host
// code the array's name is only a host-side handle, so its device address is looked up once per
// device (with that device current) and handed to kda_chunk_fwd as the workspace.  The address
// belongs to the device's current context: if that context is destroyed and re-created (a
// cudaDeviceReset, for instance), the module is loaded again at another address, so the cached
// address is keyed on the context's unique id as well and looked up again when the id changes.
#include <cuda.h>

#include <mutex>

#include "kda_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_kda_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read).  The runtime has
// made the device's primary context current by the time this runs (cudaGetDevice and
// cudaGetSymbolAddress initialise it).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {  // under g_mu
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    (void)cudaGetLastError();
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

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
    // (an id of 0, if the driver cannot report one, means: look the address up on every call)
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_kda_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
      g_scratch_ptr[dev] = p;
      g_scratch_ctx[dev] = current_context_id();
    }
    ptr = g_scratch_ptr[dev];
  }
  kda_chunk_args a = *args;
  a.workspace = ptr;
  a.workspace_bytes = KDA_NOALLOC_SCRATCH_BYTES;
  if (error_word) *error_word = ptr;
  return kda_chunk_fwd(&a, cuda_stream);
}
