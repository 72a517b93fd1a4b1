// Shared device helpers for the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Per-step log-retention floor: alpha = 0 (or a denormal) becomes e^-80.
constexpr float kLogAlphaFloor = -80.0f;

// Load element idx of a tensor whose element type is chosen at run time
// (uniform across the launch, so the branch costs nothing).
__device__ __forceinline__ float ld_elem(const void *p, size_t idx, int is_bf16)
{
    if (is_bf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[idx]);
    return reinterpret_cast<const float *>(p)[idx];
}

__device__ __forceinline__ void st_elem(void *p, size_t idx, float x, int is_bf16)
{
    if (is_bf16)
        reinterpret_cast<__nv_bfloat16 *>(p)[idx] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<float *>(p)[idx] = x;
}

__device__ __forceinline__ float log_alpha(float a)
{
    // log of the retention factor, clamped so alpha = 0 stays finite
    return fmaxf(__logf(fmaxf(a, 1e-38f)), kLogAlphaFloor);
}

// Fused input preprocessing.  Gate logit x: log alpha = -softplus(x) <= 0, clamped
// like log_alpha; beta logit y: beta = sigmoid(y); a row is scaled by 1/||row||
// (0 for a zero row).
__device__ __forceinline__ float log_alpha_from_logit(float x)
{
    return fmaxf(-(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)))), kLogAlphaFloor);
}

__device__ __forceinline__ float sigmoid_of(float y)
{
    const float e = expf(-fabsf(y));
    const float s = 1.f / (1.f + e);
    return y >= 0.f ? s : e * s;
}

__device__ __forceinline__ float inv_norm(float sum_sq)
{
    return sum_sq > 0.f ? rsqrtf(sum_sq) : 0.f;
}

__device__ __forceinline__ float4 ld_f4(const float *p)
{
    return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ void st_f4(float *p, float4 v)
{
    *reinterpret_cast<float4 *>(p) = v;
}

// Streaming variants for data touched exactly once (decode state).
__device__ __forceinline__ float4 ld_f4_stream(const float *p)
{
    return __ldcs(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ void st_f4_stream(float *p, float4 v)
{
    __stcs(reinterpret_cast<float4 *>(p), v);
}

}  // namespace kda
