// kda_forward_noalloc: the prefill for callers that cannot allocate device
// memory themselves.
//
// kda_forward needs a small caller-provided workspace: the kernel records in it
// whether one of its bounded waits gave up.  Some callers cannot provide one --
// code that runs inside an allocator-less host runtime, a plugin loaded into a
// process whose memory pool it must not touch, or a caller that has no
// allocation API at hand -- so this entry point takes only the inputs and
// outputs and uses scratch that the library itself owns: a fixed array in this
// file, kKdaNoAllocScratchBytes bytes, held on every GPU that loads the library
// until the process exits.
//
// Caveats a caller must respect:
//  * Every call shares that one array (per device), and each call clears it at
//    its start: calls that overlap on the GPU (on different streams, or from
//    different host threads without ordering) race on it.  Serialize them.
//  * The first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (a one-time set-up per device, made with that device
//    current).  Make that first call before any stream capture begins.
//  * The status word the kernel records in that array (a bounded wait that gave
//    up, invalid offsets) is read back with kda_noalloc_status(), which reads
//    the same array: call it after the call it should report on and before the
//    next kda_forward_noalloc on that device, since each call clears it.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kKdaNoAllocScratchBytes = 256;
constexpr int kMaxDevices = 64;

// Device scratch owned by the library (one copy per GPU that loads it).  In
// host code this name is only a stand-in for the symbol: its device address
// comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[kKdaNoAllocScratchBytes];

std::mutex g_setup_lock;
void *g_scratch_ptr[kMaxDevices] = {};

// The device address of the scratch array on the current device, looked up
// once per device.  Returns nullptr on failure.
void *scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> guard(g_setup_lock);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_kda_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                                          const void *alpha, const void *beta,
                                          const float *initial_state, void *o, float *final_state,
                                          int B, int T, int H, int d_k, int d_v, float scale,
                                          kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                          kda_dtype out_dtype, cudaStream_t stream)
{
    // the scratch this call needs must fit the library's array
    const size_t need = kda_forward_workspace_bytes(B, T, H, d_k, d_v);
    if (need > kKdaNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
    if (B < 0 || T < 0 || H < 0) return KDA_ERR_SHAPE;
    if (B * (long long)H == 0) return KDA_OK;
    void *scratch = scratch_for_current_device();
    if (!scratch) return KDA_ERR_LAUNCH;
    return kda_forward(q, k, v, alpha, beta, initial_state, o, final_state, B, T, H, d_k, d_v, scale,
                       qkv_dtype, gate_dtype, out_dtype, scratch, kKdaNoAllocScratchBytes, stream);
}

extern "C" kda_status kda_noalloc_status(cudaStream_t stream)
{
    void *scratch = scratch_for_current_device();
    if (!scratch) return KDA_ERR_LAUNCH;
    return kda_workspace_status(scratch, stream);
}
