// Tensor-core (tcgen05) chunked prefill. Not available in this build yet:
// every request falls back to the fp32 SIMT chunk kernel via the dispatcher.
#include "common.cuh"

namespace gdn2 {

bool chunk_tc_supported(const ChunkArgs&, int) { return false; }
size_t chunk_tc_workspace(const ChunkArgs&) { return 0; }
cudaError_t launch_chunk_tc(const ChunkArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn2
