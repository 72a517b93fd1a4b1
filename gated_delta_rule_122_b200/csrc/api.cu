// C ABI of the KDA library: argument checks on the host, then one launch on the
// caller's stream.  Nothing here allocates, synchronizes or throws.
#include <stdint.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"


namespace {

constexpr size_t kKdaWorkspaceBytes = 16;   // device status word (+ padding)

// The process-wide prefill schedule (kda_set_schedule).
std::atomic<int> g_schedule{KDA_SCHEDULE_AUTO};

bool head_size_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }
bool dtype_ok(kda_dtype t) { return t == KDA_F32 || t == KDA_BF16; }
size_t dsize(kda_dtype t) { return t == KDA_BF16 ? 2 : 4; }
bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }
bool aligned_to(const void *p, size_t n) { return p == nullptr || ((uintptr_t)p % n) == 0; }

struct Range {
    uintptr_t lo, hi;
};
Range range_of(const void *p, size_t bytes) { return Range{(uintptr_t)p, (uintptr_t)p + bytes}; }
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

// Common checks of the prefill-shaped entry points.  Sizes are in elements.
kda_status check_forward(const void *q, const void *k, const void *v, const void *alpha,
                         const void *beta, const float *s_in, const void *o, const float *s_out,
                         int B, int T, int H, int dk, int dv, kda_dtype qkv, kda_dtype gate,
                         kda_dtype out, bool gate_per_head = false)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return KDA_ERR_SHAPE;
    if (!dtype_ok(qkv) || !dtype_ok(gate) || !dtype_ok(out)) return KDA_ERR_DTYPE;
    if (!head_size_ok(dk) || !head_size_ok(dv)) return KDA_ERR_UNSUPPORTED;
    const unsigned long long tokens = (unsigned long long)B * T * H;
    if (tokens * (unsigned long long)(dk > dv ? dk : dv) >= (1ull << 62)) return KDA_ERR_SHAPE;
    if (B * (long long)H == 0) return KDA_OK;
    if (T > 0 && (!q || !k || !v || !alpha || !beta || !o)) return KDA_ERR_NULL;
    // vector tensors: 16-byte aligned rows; beta (one scalar per token): element-aligned
    // (a per-head alpha, like beta, has one scalar per token)
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
        !(gate_per_head ? aligned_to(alpha, dsize(gate)) : aligned16(alpha)) ||
        !aligned_to(beta, dsize(gate)) || !aligned16(s_in) || !aligned16(o) || !aligned16(s_out))
        return KDA_ERR_ALIGN;
    if (T > 0) {
        const Range ro = range_of(o, tokens * dv * dsize(out));
        const Range ins[] = {range_of(q, tokens * dk * dsize(qkv)), range_of(k, tokens * dk * dsize(qkv)),
                             range_of(v, tokens * dv * dsize(qkv)),
                             range_of(alpha, tokens * (gate_per_head ? 1 : dk) * dsize(gate)),
                             range_of(beta, tokens * dsize(gate)),
                             range_of(s_in, s_in ? (size_t)B * H * dk * dv * 4 : 0),
                             range_of(s_out, s_out ? (size_t)B * H * dk * dv * 4 : 0)};
        for (const Range &r : ins)
            if (overlap(ro, r)) return KDA_ERR_ALIAS;
    }
    return KDA_OK;
}

constexpr int kVarlenKda = 0, kVarlenRaw = 1, kVarlenGdn2 = 2;
kda_status check_gdn2(const void *q, const void *k, const void *v, const void *alpha, const void *erase,
                      const void *wgate, const float *s_in, const void *o, const float *s_out, int B, int T, int H,
                      int dk, int dv, kda_dtype qkv, kda_dtype gate, kda_dtype out);

// T = 0: the final state is the initial state (or zeros).
kda_status empty_sequence(const float *s_in, float *s_out, int B, int H, int dk, int dv,
                          cudaStream_t stream)
{
    if (!s_out || B * (long long)H == 0) return KDA_OK;
    const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
    cudaError_t err = cudaSuccess;
    if (!s_in)
        err = cudaMemsetAsync(s_out, 0, bytes, stream);
    else if (s_in != s_out)
        err = cudaMemcpyAsync(s_out, s_in, bytes, cudaMemcpyDeviceToDevice, stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

}  // namespace

namespace kda {

// The dense prefill variants after the workspace handling: argument checks, T = 0, and
// the launch on the tensor-core or CUDA-core kernel.  status: the device status word
// (already cleared by the caller) or null.
kda_status prefill_launch(int kind, const void *q, const void *k, const void *v, const void *alpha,
                          const void *beta, const float *initial_state, void *o, float *final_state, int B,
                          int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                          kda_dtype out_dtype, unsigned int *status, cudaStream_t stream)
{
    const bool per_head = kind == KDA_HOST_SCALAR_GATE;
    kda_status st = check_forward(q, k, v, alpha, beta, initial_state, o, final_state, B, T, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype, per_head);
    if (st != KDA_OK) return st;
    if (B * (long long)H == 0) return KDA_OK;
    if (T == 0) return empty_sequence(initial_state, final_state, B, H, d_k, d_v, stream);
    ChunkArgs a{q, k, v, alpha, beta, initial_state, final_state, o, B, T, H, scale,
                qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16, status};
    a.gate_per_head = per_head ? 1 : 0;
    a.raw_inputs = kind == KDA_HOST_RAW ? 1 : 0;
    return launch_prefill(a, d_k, d_v, qkv_dtype, gate_dtype, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

cudaError_t launch_prefill(const ChunkArgs &a, int dk, int dv, kda_dtype qkv, kda_dtype gate, cudaStream_t s)
{
    const int sched = g_schedule.load(std::memory_order_relaxed);
    const bool tc = chunk_tc_supported(dk, dv, qkv, gate);
    if (sched != KDA_SCHEDULE_CHUNKED && scan_supported(a) &&
        (sched == KDA_SCHEDULE_SCAN || scan_preferred(a, dk, dv, tc)))
        return launch_scan(a, dk, dv, s);
    return tc ? launch_chunk_tc(a, dk, dv, s) : launch_chunk_simt(a, dk, dv, s);
}

}  // namespace kda

namespace {

// Workspace handling of the dense prefill entry points: size and alignment, the status
// word cleared on the stream, then the launch.
kda_status prefill_with_workspace(int kind, const void *q, const void *k, const void *v, const void *alpha,
                                  const void *beta, const float *initial_state, void *o, float *final_state,
                                  int B, int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                                  kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream)
{
    kda_status st = check_forward(q, k, v, alpha, beta, initial_state, o, final_state, B, T, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype, kind == KDA_HOST_SCALAR_GATE);
    if (st != KDA_OK) return st;
    if (B * (long long)H == 0) return KDA_OK;
    const size_t need = kda_forward_workspace_bytes(B, T, H, d_k, d_v);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KDA_ERR_ALIGN;
    if (cudaMemsetAsync(workspace, 0, need, stream) != cudaSuccess) return KDA_ERR_LAUNCH;
    return kda::prefill_launch(kind, q, k, v, alpha, beta, initial_state, o, final_state, B, T, H, d_k, d_v, scale,
                               qkv_dtype, gate_dtype, out_dtype, static_cast<unsigned int *>(workspace), stream);
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s)
{
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_NULL: return "a required pointer is NULL";
    case KDA_ERR_SHAPE: return "a size is negative or too large";
    case KDA_ERR_DTYPE: return "unknown dtype code";
    case KDA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case KDA_ERR_UNSUPPORTED: return "head size must be a multiple of 16 from 16 to 128";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_LAUNCH: return "CUDA launch failed";
    case KDA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case KDA_ERR_ALIAS: return "an output overlaps an input";
    case KDA_ERR_VALUE: return "an enumerated argument has an unknown value";
    }
    return "unknown status";
}

int kda_version(void) { return 100; }

kda_status kda_set_schedule(int schedule)
{
    if (schedule != KDA_SCHEDULE_AUTO && schedule != KDA_SCHEDULE_CHUNKED && schedule != KDA_SCHEDULE_SCAN)
        return KDA_ERR_VALUE;
    g_schedule.store(schedule, std::memory_order_relaxed);
    return KDA_OK;
}

int kda_get_schedule(void) { return g_schedule.load(std::memory_order_relaxed); }

size_t kda_forward_workspace_bytes(int B, int T, int H, int d_k, int d_v)
{
    (void)B; (void)T; (void)H; (void)d_k; (void)d_v;
    return kKdaWorkspaceBytes;
}

kda_status kda_workspace_status(const void *workspace, cudaStream_t stream)
{
    if (!workspace) return KDA_ERR_NULL;
    if (!aligned16(workspace)) return KDA_ERR_ALIGN;
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return KDA_ERR_LAUNCH;
    if (word & 2u) return KDA_ERR_SHAPE;     // invalid sequence offsets (packed layout)
    return word ? KDA_ERR_TIMEOUT : KDA_OK;
}

kda_status kda_forward(const void *q, const void *k, const void *v, const void *alpha,
                       const void *beta, const float *initial_state, void *o, float *final_state,
                       int B, int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                       kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream)
{
    return prefill_with_workspace(KDA_HOST_FORWARD, q, k, v, alpha, beta, initial_state, o, final_state, B, T, H,
                                  d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace, workspace_bytes,
                                  stream);
}

}  // extern "C"

namespace {

// The packed-sequence prefill for every kind (KDA, raw inputs, GDN-2): checks, workspace,
// then the launch.  For GDN-2, `beta` is the erase gate and `wgate` the write gate.
kda_status varlen_prefill(int kind, const void *q, const void *k, const void *v, const void *alpha,
                          const void *beta, const void *wgate, const int *cu_seqlens, const float *initial_state,
                          void *o, float *final_state, int N, int total_T, int H, int d_k, int d_v, float scale,
                          kda_dtype qkv_dtype, kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream)
{
    if (N < 0) return KDA_ERR_SHAPE;
    const bool gdn2 = kind == kVarlenGdn2;
    // the token tensors are one [1, total_T, H, d] batch; the states are per sequence
    kda_status st = gdn2 ? check_gdn2(q, k, v, alpha, beta, wgate, nullptr, o, nullptr, 1, total_T, H, d_k, d_v,
                                      qkv_dtype, gate_dtype, out_dtype)
                         : check_forward(q, k, v, alpha, beta, nullptr, o, nullptr, 1, total_T, H, d_k, d_v,
                                         qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (N * (long long)H == 0) return KDA_OK;
    if (!cu_seqlens) return KDA_ERR_NULL;
    if (!aligned_to(cu_seqlens, sizeof(int)) || !aligned16(initial_state) || !aligned16(final_state))
        return KDA_ERR_ALIGN;
    if ((unsigned long long)N * H * d_k * d_v >= (1ull << 60)) return KDA_ERR_SHAPE;
    if (total_T > 0) {
        const size_t state_bytes = (size_t)N * H * d_k * d_v * 4;
        const Range ro = range_of(o, (size_t)total_T * H * d_v * dsize(out_dtype));
        if (overlap(ro, range_of(initial_state, initial_state ? state_bytes : 0)) ||
            overlap(ro, range_of(final_state, final_state ? state_bytes : 0)) ||
            overlap(ro, range_of(cu_seqlens, (size_t)(N + 1) * sizeof(int))))
            return KDA_ERR_ALIAS;
    }
    const size_t need = kda_forward_workspace_bytes(N, total_T, H, d_k, d_v);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KDA_ERR_ALIGN;
    if (cudaMemsetAsync(workspace, 0, need, stream) != cudaSuccess) return KDA_ERR_LAUNCH;
    // no tokens at all: every sequence is empty (the offsets are all zero)
    if (total_T == 0) return empty_sequence(initial_state, final_state, N, H, d_k, d_v, stream);
    kda::ChunkArgs a{q, k, v, alpha, gdn2 ? nullptr : beta, initial_state, final_state, o, N, total_T, H, scale,
                     qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                     static_cast<unsigned int *>(workspace), cu_seqlens};
    if (gdn2) {
        a.erase = beta;
        a.wgate = wgate;
    }
    a.raw_inputs = kind == kVarlenRaw ? 1 : 0;
    return kda::launch_prefill(a, d_k, d_v, qkv_dtype, gate_dtype, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

}  // namespace

extern "C" {

kda_status kda_forward_varlen(const void *q, const void *k, const void *v, const void *alpha,
                              const void *beta, const int *cu_seqlens, const float *initial_state,
                              void *o, float *final_state, int N, int total_T, int H, int d_k,
                              int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                              kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream)
{
    return varlen_prefill(kVarlenKda, q, k, v, alpha, beta, nullptr, cu_seqlens, initial_state, o, final_state, N,
                          total_T, H, d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace, workspace_bytes,
                          stream);
}

kda_status kda_forward_varlen_raw(const void *q, const void *k, const void *v, const void *gate_logit,
                                  const void *beta_logit, const int *cu_seqlens, const float *initial_state,
                                  void *o, float *final_state, int N, int total_T, int H, int d_k, int d_v,
                                  float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype, kda_dtype out_dtype,
                                  void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return varlen_prefill(kVarlenRaw, q, k, v, gate_logit, beta_logit, nullptr, cu_seqlens, initial_state, o,
                          final_state, N, total_T, H, d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace,
                          workspace_bytes, stream);
}

kda_status kda_forward_varlen_gdn2(const void *q, const void *k, const void *v, const void *alpha,
                                   const void *erase, const void *write, const int *cu_seqlens,
                                   const float *initial_state, void *o, float *final_state, int N, int total_T,
                                   int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                   kda_dtype out_dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    return varlen_prefill(kVarlenGdn2, q, k, v, alpha, erase, write, cu_seqlens, initial_state, o, final_state, N,
                          total_T, H, d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace, workspace_bytes,
                          stream);
}

kda_status kda_forward_scalar_gate(const void *q, const void *k, const void *v, const void *alpha,
                                   const void *beta, const float *initial_state, void *o,
                                   float *final_state, int B, int T, int H, int d_k, int d_v,
                                   float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                   kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream)
{
    return prefill_with_workspace(KDA_HOST_SCALAR_GATE, q, k, v, alpha, beta, initial_state, o, final_state, B, T,
                                  H, d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace, workspace_bytes,
                                  stream);
}

kda_status kda_forward_raw(const void *q, const void *k, const void *v, const void *gate_logit,
                           const void *beta_logit, const float *initial_state, void *o, float *final_state,
                           int B, int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                           kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream)
{
    return prefill_with_workspace(KDA_HOST_RAW, q, k, v, gate_logit, beta_logit, initial_state, o, final_state, B,
                                  T, H, d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype, workspace,
                                  workspace_bytes, stream);
}

kda_status kda_decode_step_raw(const void *q, const void *k, const void *v, const void *gate_logit,
                               const void *beta_logit, float *state, void *o, int N, int H, int d_k,
                               int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                               kda_dtype out_dtype, cudaStream_t stream)
{
    if (N * (long long)H > 0 && !state) return KDA_ERR_NULL;
    kda_status st = check_forward(q, k, v, gate_logit, beta_logit, state, o, nullptr, N, 1, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (N * (long long)H == 0) return KDA_OK;
    kda::RecurrentArgs a{q, k, v, gate_logit, beta_logit, state, state, o, N, 1, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16, nullptr};
    a.raw_inputs = 1;
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

}  // extern "C"

namespace {

// GDN-2 entry points: the erase and write gates take the place of beta.
kda_status check_gdn2(const void *q, const void *k, const void *v, const void *alpha,
                             const void *erase, const void *wgate, const float *s_in, const void *o,
                             const float *s_out, int B, int T, int H, int dk, int dv, kda_dtype qkv,
                             kda_dtype gate, kda_dtype out)
{
    // erase stands in for beta in the common checks (presence, alignment, aliasing of o)
    kda_status st = check_forward(q, k, v, alpha, erase, s_in, o, s_out, B, T, H, dk, dv, qkv, gate, out);
    if (st != KDA_OK) return st;
    if (B * (long long)H == 0 || T == 0) return KDA_OK;
    if (!wgate) return KDA_ERR_NULL;
    if (!aligned16(erase) || !aligned16(wgate)) return KDA_ERR_ALIGN;
    const unsigned long long tokens = (unsigned long long)B * T * H;
    const Range ro = range_of(o, tokens * dv * dsize(out));
    if (overlap(ro, range_of(erase, tokens * dk * dsize(gate))) ||
        overlap(ro, range_of(wgate, tokens * dv * dsize(gate))))
        return KDA_ERR_ALIAS;
    return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_forward_gdn2(const void *q, const void *k, const void *v, const void *alpha,
                            const void *erase, const void *wgate, const float *initial_state, void *o,
                            float *final_state, int B, int T, int H, int d_k, int d_v, float scale,
                            kda_dtype qkv_dtype, kda_dtype gate_dtype, kda_dtype out_dtype,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    kda_status st = check_gdn2(q, k, v, alpha, erase, wgate, initial_state, o, final_state, B, T, H,
                               d_k, d_v, qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (B * (long long)H == 0) return KDA_OK;
    const size_t need = kda_forward_workspace_bytes(B, T, H, d_k, d_v);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KDA_ERR_ALIGN;
    if (cudaMemsetAsync(workspace, 0, need, stream) != cudaSuccess) return KDA_ERR_LAUNCH;
    if (T == 0) return empty_sequence(initial_state, final_state, B, H, d_k, d_v, stream);
    kda::ChunkArgs a{q, k, v, alpha, nullptr, initial_state, final_state, o, B, T, H, scale,
                     qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                     static_cast<unsigned int *>(workspace), nullptr, 0, erase, wgate};
    // the tensor-core kernel for d_k = d_v = 128 with bf16 inputs and gates, the CUDA-core
    // chunk kernel for every other shape and dtype
    cudaError_t err;
    if (kda::chunk_tc_supported(d_k, d_v, qkv_dtype, gate_dtype))
        err = kda::launch_chunk_tc(a, d_k, d_v, stream);
    else
        err = kda::launch_chunk_simt(a, d_k, d_v, stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_forward_sequential(const void *q, const void *k, const void *v, const void *alpha,
                                  const void *beta, const float *initial_state, void *o,
                                  float *final_state, int B, int T, int H, int d_k, int d_v,
                                  float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                  kda_dtype out_dtype, cudaStream_t stream)
{
    kda_status st = check_forward(q, k, v, alpha, beta, initial_state, o, final_state, B, T, H,
                                  d_k, d_v, qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (B * (long long)H == 0) return KDA_OK;
    if (T == 0) return empty_sequence(initial_state, final_state, B, H, d_k, d_v, stream);
    kda::RecurrentArgs a{q, k, v, alpha, beta, initial_state, final_state, o, B, T, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                         nullptr};
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *alpha,
                           const void *beta, float *state, void *o, int N, int H, int d_k,
                           int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                           kda_dtype out_dtype, cudaStream_t stream)
{
    if (N * (long long)H > 0 && !state) return KDA_ERR_NULL;
    kda_status st = check_forward(q, k, v, alpha, beta, state, o, nullptr, N, 1, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (N * (long long)H == 0) return KDA_OK;
    // the state is read and rewritten in place; one token per sequence
    kda::RecurrentArgs a{q, k, v, alpha, beta, state, state, o, N, 1, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                         nullptr};
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_decode_step_scalar_gate(const void *q, const void *k, const void *v,
                                       const void *alpha, const void *beta, float *state, void *o,
                                       int N, int H, int d_k, int d_v, float scale,
                                       kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                       kda_dtype out_dtype, cudaStream_t stream)
{
    if (N * (long long)H > 0 && !state) return KDA_ERR_NULL;
    kda_status st = check_forward(q, k, v, alpha, beta, state, o, nullptr, N, 1, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype, true);
    if (st != KDA_OK) return st;
    if (N * (long long)H == 0) return KDA_OK;
    kda::RecurrentArgs a{q, k, v, alpha, beta, state, state, o, N, 1, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                         nullptr, nullptr, 1};
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_decode_step_gdn2(const void *q, const void *k, const void *v, const void *alpha,
                                const void *erase, const void *wgate, float *state, void *o, int N,
                                int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                                kda_dtype gate_dtype, kda_dtype out_dtype, cudaStream_t stream)
{
    if (N * (long long)H > 0 && !state) return KDA_ERR_NULL;
    kda_status st = check_gdn2(q, k, v, alpha, erase, wgate, state, o, nullptr, N, 1, H, d_k, d_v,
                               qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (N * (long long)H == 0) return KDA_OK;
    kda::RecurrentArgs a{q, k, v, alpha, nullptr, state, state, o, N, 1, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                         nullptr, nullptr, 0, erase, wgate};
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_decode_tokens(const void *q, const void *k, const void *v, const void *alpha,
                             const void *beta, float *state, const int *state_slots, int num_slots,
                             int commit, float *token_states, void *o, int N, int T, int H, int d_k,
                             int d_v, float scale, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                             kda_dtype out_dtype, void *status, cudaStream_t stream)
{
    kda_status st = check_forward(q, k, v, alpha, beta, nullptr, o, nullptr, N, T, H, d_k, d_v,
                                  qkv_dtype, gate_dtype, out_dtype);
    if (st != KDA_OK) return st;
    if (num_slots < 0 || (!state_slots && num_slots < N)) return KDA_ERR_SHAPE;
    if (!aligned16(state) || !aligned16(token_states) || !aligned16(status) ||
        !aligned_to(state_slots, sizeof(int)))
        return KDA_ERR_ALIGN;
    if (status && cudaMemsetAsync(status, 0, sizeof(unsigned int), stream) != cudaSuccess)
        return KDA_ERR_LAUNCH;
    if (N * (long long)H == 0 || T == 0) return KDA_OK;
    if (!state) return KDA_ERR_NULL;
    const size_t per_state = (size_t)H * d_k * d_v * sizeof(float);
    const Range ro = range_of(o, (size_t)N * T * H * d_v * dsize(out_dtype));
    const Range rp = range_of(state, (size_t)num_slots * per_state);
    const Range rt = range_of(token_states, token_states ? (size_t)N * T * per_state : 0);
    if (overlap(ro, rp) || overlap(ro, rt) || overlap(rp, rt)) return KDA_ERR_ALIAS;
    kda::RecurrentArgs a{q, k, v, alpha, beta, state, commit ? state : nullptr, o, N, T, H, scale,
                         qkv_dtype == KDA_BF16, gate_dtype == KDA_BF16, out_dtype == KDA_BF16,
                         static_cast<unsigned int *>(status)};
    a.state_slots = state_slots;
    a.num_slots = num_slots;
    a.token_states = token_states;
    return kda::launch_recurrent(a, d_k, d_v, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_state_copy(const float *src, const int *src_index, int src_slots, float *dst,
                          const int *dst_index, int dst_slots, int count, int H, int d_k, int d_v,
                          void *status, cudaStream_t stream)
{
    if (count < 0 || src_slots < 0 || dst_slots < 0 || H < 0) return KDA_ERR_SHAPE;
    if (!head_size_ok(d_k) || !head_size_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if ((!src_index && count > src_slots) || (!dst_index && count > dst_slots)) return KDA_ERR_SHAPE;
    if (!aligned16(src) || !aligned16(dst) || !aligned16(status) || !aligned_to(src_index, sizeof(int)) ||
        !aligned_to(dst_index, sizeof(int)))
        return KDA_ERR_ALIGN;
    if (status && cudaMemsetAsync(status, 0, sizeof(unsigned int), stream) != cudaSuccess)
        return KDA_ERR_LAUNCH;
    if (count == 0 || H == 0) return KDA_OK;
    if (!src || !dst) return KDA_ERR_NULL;
    kda::StateCopyArgs a{src, src_index, src_slots, dst, dst_index, dst_slots, count,
                         (size_t)H * d_k * d_v / 4, static_cast<unsigned int *>(status)};
    return kda::launch_state_copy(a, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

kda_status kda_selftest_bounded_wait(int arrive, unsigned int limit_us, void *status, cudaStream_t stream)
{
    if (!status) return KDA_ERR_NULL;
    if (!aligned16(status)) return KDA_ERR_ALIGN;
    if (limit_us == 0 || limit_us > 2000000u) return KDA_ERR_SHAPE;
    if (cudaMemsetAsync(status, 0, sizeof(unsigned int), stream) != cudaSuccess) return KDA_ERR_LAUNCH;
    return kda::launch_bounded_wait_selftest(arrive, 1000ull * limit_us, static_cast<unsigned int *>(status),
                                             stream) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_LAUNCH;
}

}  // extern "C"
