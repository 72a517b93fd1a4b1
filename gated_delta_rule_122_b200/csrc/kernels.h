// Launch interfaces shared by the C ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>

#include "../../include/kda.h"

namespace kda {

// Arguments of every prefill-shaped launch (also the decode step, with T = 1).
struct ChunkArgs {
    const void *q, *k, *v, *alpha, *beta;
    const float *s_in;   // [B,H,DK,DV] fp32 or null (zero state)
    float *s_out;        // [B,H,DK,DV] fp32 or null; may equal s_in
    void *o;             // [B,T,H,DV]
    int B, T, H;
    float scale;
    int qkv_bf16, gate_bf16, out_bf16;
    unsigned int *status;   // device status word (bit 0: a bounded wait timed out) or null
};
using RecurrentArgs = ChunkArgs;

cudaError_t launch_recurrent(const RecurrentArgs &a, int dk, int dv, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs &a, int dk, int dv, cudaStream_t s);
bool chunk_tc_supported(int dk, int dv, kda_dtype qkv, kda_dtype gate);
cudaError_t launch_chunk_tc(const ChunkArgs &a, int dk, int dv, cudaStream_t s);

}  // namespace kda
