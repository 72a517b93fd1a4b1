// Instances of the column-scan prefill for key sizes 80, 96, 112, 128 (compiled apart so that
// the instances build in parallel).
#include "scan.cuh"

namespace kda {
namespace scan {

template cudaError_t launch_scan_dk<80>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<96>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<112>(const ChunkArgs &, int, cudaStream_t);
template cudaError_t launch_scan_dk<128>(const ChunkArgs &, int, cudaStream_t);

}  // namespace scan
}  // namespace kda
