// Whole-state copies between slot pools: the serving operations that duplicate or
// restore a sequence's recurrent state (fork, prefix sharing, rollback of a
// speculative step, migration between pools).  A state is request-scoped like a
// KV-cache slot and must be copied whenever a request is duplicated or rewound:
// "Module 03 -- KDA I: The Delta-Rule Recurrence", section 5 "State vs.
// checkpoint weights".
//
// The copy is a pure HBM stream: each entry moves one [H, DK, DV] fp32 block
// (4 MiB at H = 64, d = 128).  Blocks of 256 threads each move 16-byte vectors
// with four loads in flight per thread; the grid covers every entry with about
// eight blocks per SM in total, each entry split into equal pieces.
#include "common.cuh"
#include "kernels.h"

namespace kda {

namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads)
kda_state_copy_kernel(StateCopyArgs a)
{
    for (int i = blockIdx.y; i < a.count; i += gridDim.y) {
        const int si = a.src_index ? a.src_index[i] : i;
        const int di = a.dst_index ? a.dst_index[i] : i;
        if (si < 0 || di < 0) continue;   // a skipped entry
        if (si >= a.src_slots || di >= a.dst_slots) {
            if (a.status && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.status, 2u);
            continue;
        }
        const float4 *src = reinterpret_cast<const float4 *>(a.src) + (size_t)si * a.vec_per_state;
        float4 *dst = reinterpret_cast<float4 *>(a.dst) + (size_t)di * a.vec_per_state;
        const size_t stride = (size_t)gridDim.x * kCopyThreads;
        size_t j = (size_t)blockIdx.x * kCopyThreads + threadIdx.x;
        for (; j + (kCopyUnroll - 1) * stride < a.vec_per_state; j += kCopyUnroll * stride) {
            float4 x[kCopyUnroll];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) x[u] = __ldcs(src + j + u * stride);
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) __stcs(dst + j + u * stride, x[u]);
        }
        for (; j < a.vec_per_state; j += stride) __stcs(dst + j, __ldcs(src + j));
    }
}

}  // namespace

cudaError_t launch_state_copy(const StateCopyArgs &a, cudaStream_t stream)
{
    if (a.count <= 0 || a.vec_per_state == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned gy = (unsigned)(a.count < 65535 ? a.count : 65535);
    const long long target = 8LL * sms;   // resident blocks over the whole grid
    long long gx = (target + gy - 1) / gy;
    const long long most = (long long)((a.vec_per_state + kCopyThreads - 1) / kCopyThreads);
    if (gx > most) gx = most;
    if (gx < 1) gx = 1;
    kda_state_copy_kernel<<<dim3((unsigned)gx, gy), kCopyThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
