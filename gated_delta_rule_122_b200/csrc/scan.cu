// Dispatch of the column-scan prefill over the key size, and the rule that picks it; the
// kernel template is in scan.cuh.
#include "scan.cuh"

namespace kda {
namespace scan {
extern template cudaError_t launch_scan_dk<16>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<32>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<48>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<64>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<80>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<96>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<112>(const ChunkArgs &, int, cudaStream_t);
extern template cudaError_t launch_scan_dk<128>(const ChunkArgs &, int, cudaStream_t);
}  // namespace scan

bool scan_supported(const ChunkArgs &a)
{
    return !a.raw_inputs && !a.erase && !a.wgate && !a.state_slots && !a.token_states;
}

// Measured on a B200 (T = 2048, CUDA events): the scan is faster than the CUDA-core chunk
// kernel at every size tried (d = 64: 4 heads 0.37 against 1.32 ms, 1184 heads 4.4
// against 12.5 ms; d = 128 fp32: 128 heads 2.7 against 3.5 ms; d = 16: 0.25 against
// 0.37 ms), and slower than the tensor-core chunk kernel even for few heads (d = 128
// bf16, 4 heads: 0.46 against 0.24 ms).  So the scan replaces the CUDA-core chunk kernel
// wherever it applies and never the tensor-core one.
bool scan_preferred(const ChunkArgs &a, int dk, int dv, bool tc)
{
    (void)dk;
    (void)dv;
    return scan_supported(a) && !tc;
}

cudaError_t launch_scan(const ChunkArgs &a, int dk, int dv, cudaStream_t s)
{
    if (!scan_supported(a) || dv % 16 != 0) return cudaErrorInvalidValue;
    switch (dk) {
    case 16: return scan::launch_scan_dk<16>(a, dv, s);
    case 32: return scan::launch_scan_dk<32>(a, dv, s);
    case 48: return scan::launch_scan_dk<48>(a, dv, s);
    case 64: return scan::launch_scan_dk<64>(a, dv, s);
    case 80: return scan::launch_scan_dk<80>(a, dv, s);
    case 96: return scan::launch_scan_dk<96>(a, dv, s);
    case 112: return scan::launch_scan_dk<112>(a, dv, s);
    case 128: return scan::launch_scan_dk<128>(a, dv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
