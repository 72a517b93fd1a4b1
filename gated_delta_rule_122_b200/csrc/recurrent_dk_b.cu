// Instances of the token-by-token kernel for key sizes 80, 96, 112, 128 (compiled apart so that
// the instances build in parallel).
#include "recurrent.cuh"

namespace kda {

template cudaError_t launch_recurrent_dk<80>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<96>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<112>(const RecurrentArgs &, int, cudaStream_t);
template cudaError_t launch_recurrent_dk<128>(const RecurrentArgs &, int, cudaStream_t);

}  // namespace kda
