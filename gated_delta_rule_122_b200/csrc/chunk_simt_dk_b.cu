// Instances of the CUDA-core chunk kernel for key sizes 48 and 64 (compiled apart so that
// the instances build in parallel).
#include "chunk_simt.cuh"

namespace kda {

template cudaError_t launch_chunk_simt_dk<48>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_chunk_simt_dk<64>(const ChunkArgs &, int, cudaStream_t);

}  // namespace kda
