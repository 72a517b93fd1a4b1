// Instances of the token-by-token kernel for key sizes 16, 32, 48, 64 (compiled apart so that
// the instances build in parallel).
#include "recurrent.cuh"

namespace kda {

template cudaError_t launch_recurrent_dk<16>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<32>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<48>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<64>(const RecurrentArgs &, int, cudaStream_t);

}  // namespace kda
