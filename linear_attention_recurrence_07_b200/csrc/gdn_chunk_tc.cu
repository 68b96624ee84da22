// Tensor-core (tcgen05) chunkwise prefill for bf16 inputs.  Placeholder until the
// kernel lands: reports itself unavailable so bf16 prefill runs the CUDA-core kernel.
#include "gdn_internal.cuh"

namespace gdn {

bool chunk_tc_available() { return false; }

cudaError_t launch_chunk_tc(const ChunkArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
