// Instances of the column-scan prefill for key sizes 16, 32, 48, 64 (compiled apart so that
// the instances build in parallel).
#include "scan.cuh"

namespace kda {
namespace scan {

template cudaError_t launch_scan_dk<16>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<32>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<48>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<64>(const ChunkArgs &, int, cudaStream_t);

}  // namespace scan
}  // namespace kda
