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
    // GDN-2: a per-key-channel erase gate [B, T, H, d_k] and a per-value-channel write
    // gate [B, T, H, d_v] (gate dtype) in place of beta; null for KDA.
    const void *erase, *wgate;
    // Decode over a pool of state slots: sequence b reads s_in and writes s_out at
    // slot state_slots[b] (a negative slot skips the sequence; a slot >= num_slots is
    // skipped and sets status bit 1).  Null: slot b.
    const int *state_slots;
    int num_slots;
    // The state after each token, [B, T, H, DK, DV] fp32, or null.
    float *token_states;
    // Fused input preprocessing: q and k arrive un-normalised (each token's row is
    // divided by its L2 norm), alpha holds gate logits x (log alpha = -softplus(x))
    // and beta holds beta logits y (beta = sigmoid(y)).
    int raw_inputs;
};

// Where sequence b's token rows sit.  Dense tensors are [B, T, H, d] and sequence b
// owns rows b*T .. b*T+T-1; with offsets they are [1, T, H, d] (T = total tokens) and
// sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1.  Kernels index rows as
// (tok0 + t) * H + h and never derive shifted pointers.  Returns false when the
// offsets of sequence b are invalid.
struct SeqSpan {
    size_t tok0;   // the sequence's first token row
    int len;       // its number of tokens
};

__host__ __device__ inline bool sequence_span(const ChunkArgs &a, int b, SeqSpan &sp)
{
    if (!a.cu_seqlens) {
        sp.tok0 = (size_t)b * a.T;
        sp.len = a.T;
        return true;
    }
    const int s0 = a.cu_seqlens[b], s1 = a.cu_seqlens[b + 1];
    if (s0 < 0 || s1 < s0 || s1 > a.T) return false;
    sp.tok0 = (size_t)s0;
    sp.len = s1 - s0;
    return true;
}
using RecurrentArgs = ChunkArgs;

cudaError_t launch_recurrent(const RecurrentArgs &a, int dk, int dv, cudaStream_t s);

// Entry i copies the [H, DK, DV] block src[src_index[i]] to dst[dst_index[i]]
// (identity index when null; negative: skipped; out of range: skipped, status bit 1).
struct StateCopyArgs {
    const float *src;
    const int *src_index;
    int src_slots;
    float *dst;
    const int *dst_index;
    int dst_slots;
    int count;
    size_t vec_per_state;   // H * DK * DV / 4
    unsigned int *status;   // device status word or null
};
cudaError_t launch_state_copy(const StateCopyArgs &a, cudaStream_t s);
cudaError_t launch_bounded_wait_selftest(int arrive, unsigned long long limit_ns, unsigned int *status,
                                         cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs &a, int dk, int dv, cudaStream_t s);
// (both take GDN-2 gates when a.erase is set)
bool chunk_tc_supported(int dk, int dv, kda_dtype qkv, kda_dtype gate);
cudaError_t launch_chunk_tc(const ChunkArgs &a, int dk, int dv, cudaStream_t s);
// The column-scan prefill (one 8-lane group per value column, token by token): plain KDA
// and the per-head gate, no raw inputs or GDN-2 gates.  scan_preferred: the automatic
// schedule takes the scan over the chunk kernel that would run otherwise (tc: the
// tensor-core one).
bool scan_supported(const ChunkArgs &a);
bool scan_preferred(const ChunkArgs &a, int dk, int dv, bool tc);
cudaError_t launch_scan(const ChunkArgs &a, int dk, int dv, cudaStream_t s);
// The prefill launch chosen for a's variant and shape under the process-wide schedule
// setting: the column scan, the tensor-core chunk kernel or the CUDA-core one.
cudaError_t launch_prefill(const ChunkArgs &a, int dk, int dv, kda_dtype qkv, kda_dtype gate, cudaStream_t s);

// The dense prefill (kind: KDA_HOST_FORWARD, KDA_HOST_SCALAR_GATE or KDA_HOST_RAW) after
// the workspace handling: argument checks, T = 0, the launch; status cleared by the caller.
kda_status prefill_launch(int kind, const void *q, const void *k, const void *v, const void *alpha,
                          const void *beta, const float *initial_state, void *o, float *final_state, int B,
                          int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                          kda_dtype out_dtype, unsigned int *status, cudaStream_t stream);

}  // namespace kda
