// Instances of the CUDA-core chunk kernel for key sizes 16 and 32 (compiled apart so that
// the instances build in parallel).
#include "chunk_simt.cuh"

namespace kda {

template cudaError_t launch_chunk_simt_dk<16>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_chunk_simt_dk<32>(const ChunkArgs &, int, cudaStream_t);

}  // namespace kda
