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
    unsigned int *status;   // device status word (bit 0: a bounded wait timed out,
                            // bit 1: invalid sequence offsets) or null
    // Packed variable-length batch: sequence b owns token rows cu_seqlens[b] ..
    // cu_seqlens[b+1]-1 of tensors laid out [1, T, H, d] (T = total tokens).  Null
    // for the dense [B, T, H, d] layout.
    const int *cu_seqlens;
    // One retention factor per (token, head) -- Gated DeltaNet's scalar gate -- with
    // alpha laid out [B, T, H]; 0 for the per-key-channel gate [B, T, H, d_k].
    int gate_per_head;
};

// The per-sequence view of a launch: with offsets, the sequence's rows are made
// to look like a batch of one (base pointers advanced, T = its length).  Returns
// false when the offsets of sequence b are invalid.
__host__ __device__ inline bool sequence_view(const ChunkArgs &a, int b, int dk, int dv, ChunkArgs &s,
                                              int &b_local, int &row0)
{
    s = a;
    b_local = b;
    row0 = 0;
    if (!a.cu_seqlens) return true;
    const int s0 = a.cu_seqlens[b], s1 = a.cu_seqlens[b + 1];
    if (s0 < 0 || s1 < s0 || s1 > a.T) return false;
    const size_t rows = (size_t)s0 * a.H;   // token-head rows before the sequence
    const size_t qe = a.qkv_bf16 ? 2 : 4, ge = a.gate_bf16 ? 2 : 4, oe = a.out_bf16 ? 2 : 4;
    s.q = (const char *)a.q + rows * dk * qe;
    s.k = (const char *)a.k + rows * dk * qe;
    s.v = (const char *)a.v + rows * dv * qe;
    s.alpha = (const char *)a.alpha + rows * (a.gate_per_head ? 1 : dk) * ge;
    s.beta = (const char *)a.beta + rows * ge;
    s.o = (char *)a.o + rows * dv * oe;
    s.T = s1 - s0;
    b_local = 0;
    row0 = s0;
    return true;
}
using RecurrentArgs = ChunkArgs;

cudaError_t launch_recurrent(const RecurrentArgs &a, int dk, int dv, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs &a, int dk, int dv, cudaStream_t s);
bool chunk_tc_supported(int dk, int dv, kda_dtype qkv, kda_dtype gate);
cudaError_t launch_chunk_tc(const ChunkArgs &a, int dk, int dv, cudaStream_t s);

}  // namespace kda
