// Dispatch of the token-by-token kernel over the key size; the kernel template and
// its per-value-size launches are in recurrent.cuh.
#include "recurrent.cuh"

namespace kda {

extern template cudaError_t launch_recurrent_dk<16>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<32>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<48>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<64>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<80>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<96>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<112>(const RecurrentArgs &, int, cudaStream_t);
extern template cudaError_t launch_recurrent_dk<128>(const RecurrentArgs &, int, cudaStream_t);

cudaError_t launch_recurrent(const RecurrentArgs &a, int dk, int dv, cudaStream_t s)
{
    switch (dk) {
    case 16: return launch_recurrent_dk<16>(a, dv, s);
    case 32: return launch_recurrent_dk<32>(a, dv, s);
    case 48: return launch_recurrent_dk<48>(a, dv, s);
    case 64: return launch_recurrent_dk<64>(a, dv, s);
    case 80: return launch_recurrent_dk<80>(a, dv, s);
    case 96: return launch_recurrent_dk<96>(a, dv, s);
    case 112: return launch_recurrent_dk<112>(a, dv, s);
    case 128: return launch_recurrent_dk<128>(a, dv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
