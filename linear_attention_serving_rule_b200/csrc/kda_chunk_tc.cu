// kda_chunk_tc.cu -- tcgen05 tensor-core chunkwise KDA prefill (bf16, dk = dv = 128).
#include "kda_internal.cuh"

namespace kda {
cudaError_t launch_chunk_tc(const Plan&, const ChunkParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
