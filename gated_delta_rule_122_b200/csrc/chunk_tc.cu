// Tensor-core (tcgen05) chunkwise KDA prefill -- placeholder until the kernel lands.
#include "common.cuh"
#include "kernels.h"

namespace kda {
bool chunk_tc_supported(int, int, kda_dtype, kda_dtype) { return false; }
cudaError_t launch_chunk_tc(const ChunkArgs &, int, int, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
