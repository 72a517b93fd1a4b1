// Instances of the CUDA-core chunk kernel for key sizes 112 and 128 (compiled apart so that
// the instances build in parallel).
#include "chunk_simt.cuh"

namespace kda {

template cudaError_t launch_chunk_simt_dk<112>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_chunk_simt_dk<128>(const ChunkArgs &, int, cudaStream_t);

}  // namespace kda
