// kda_chunk_tc.cu -- tensor-core (tcgen05) chunkwise prefill; not built yet.
#include "kda_internal.cuh"

namespace kda {

bool chunk_tc_supported(int, int, int) { return false; }

cudaError_t launch_chunk_tc(const ChunkArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
