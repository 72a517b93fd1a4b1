// Prefill and decode with HOST buffers: the library moves the inputs in and the results
// out itself, overlapping the copies with the kernels, so a caller whose tensors live in
// host memory makes one call per operation.
//
// Prefill: the sequence is cut into segments of kSegment tokens.  Segment j's inputs are
// copied in on one stream while the kernel runs segment j-1 on the caller's stream
// (continuing from the state segment j-1 left, in place), and segment j-2's outputs are
// copied back on a third stream; two device slots per buffer make the three overlap.
// Every copy is one cudaMemcpyAsync of one contiguous host run (a sequence's rows of
// one segment).  The final state, when asked for, is copied back after the last
// segment.  Nothing here is part of the recurrence: it is the data movement of a host
// caller ("Module 03 -- KDA I: The Delta-Rule Recurrence", section 5: the state is
// per-request serving state that the caller keeps).
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kSegment = 1024;          // tokens per pipelined segment
constexpr size_t kAlign = 256;

size_t esize(kda_dtype t) { return t == KDA_BF16 ? 2 : 4; }
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool head_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }
bool dtype_ok(kda_dtype t) { return t == KDA_F32 || t == KDA_BF16; }

// Byte sizes of one device slot's buffers for a segment of L tokens.
struct SlotPlan {
    size_t q, k, v, a, b, o;
    size_t total() const { return up(q) + up(k) + up(v) + up(a) + up(b) + up(o); }
};

SlotPlan slot_plan(int B, int L, int H, int dk, int dv, kda_dtype qkv, kda_dtype gate, kda_dtype out,
                   bool gate_per_head)
{
    const size_t rows = (size_t)B * L * H;
    SlotPlan s;
    s.q = rows * dk * esize(qkv);
    s.k = s.q;
    s.v = rows * dv * esize(qkv);
    s.a = rows * (gate_per_head ? 1 : dk) * esize(gate);
    s.b = rows * esize(gate);
    s.o = rows * dv * esize(out);
    return s;
}

int segment_len(int T) { return T < kSegment ? (T > 0 ? T : 1) : kSegment; }

// A copy of sequence b's rows t0 .. t0+L-1 of a host tensor [B, T, H, width] (elements of
// esz bytes) to or from a device buffer [B, L, H, width].
cudaError_t copy_rows(void *dev, const void *host, bool to_device, int b, int T, int L, int t0, int H,
                      size_t width_bytes, cudaStream_t s)
{
    const size_t run = (size_t)L * H * width_bytes;
    char *d = static_cast<char *>(dev) + (size_t)b * run;
    const char *hsrc = static_cast<const char *>(host) + ((size_t)b * T + t0) * H * width_bytes;
    if (to_device) return cudaMemcpyAsync(d, hsrc, run, cudaMemcpyHostToDevice, s);
    return cudaMemcpyAsync(const_cast<char *>(hsrc), d, run, cudaMemcpyDeviceToHost, s);
}

}  // namespace

extern "C" {

size_t kda_forward_host_workspace_bytes(int B, int T, int H, int d_k, int d_v, kda_dtype qkv_dtype,
                                        kda_dtype gate_dtype, kda_dtype out_dtype, int kind)
{
    if (B < 0 || T < 0 || H < 0 || d_k <= 0 || d_v <= 0) return 0;
    const SlotPlan s = slot_plan(B, segment_len(T), H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype,
                                 kind == KDA_HOST_SCALAR_GATE);
    const size_t state = (size_t)B * H * d_k * d_v * 4;
    return kAlign + up(state) + 2 * s.total();
}

kda_status kda_forward_host(int kind, const void *q, const void *k, const void *v, const void *alpha,
                            const void *beta, const float *initial_state, void *o, float *final_state,
                            int B, int T, int H, int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                            kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream)
{
    if (kind != KDA_HOST_FORWARD && kind != KDA_HOST_SCALAR_GATE && kind != KDA_HOST_RAW) return KDA_ERR_SHAPE;
    if (B < 0 || T < 0 || H < 0 || d_k <= 0 || d_v <= 0) return KDA_ERR_SHAPE;
    if (!dtype_ok(qkv_dtype) || !dtype_ok(gate_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_DTYPE;
    if (!head_ok(d_k) || !head_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (B * (long long)H == 0) return KDA_OK;
    if (T > 0 && (!q || !k || !v || !alpha || !beta || !o)) return KDA_ERR_NULL;
    const bool per_head = kind == KDA_HOST_SCALAR_GATE;
    const size_t need = kda_forward_host_workspace_bytes(B, T, H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype, kind);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if ((uintptr_t)workspace % kAlign) return KDA_ERR_ALIGN;

    const int S = segment_len(T);
    const SlotPlan sp = slot_plan(B, S, H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype, per_head);
    char *ws = static_cast<char *>(workspace);
    void *status = ws;                                   // the kernel's status word
    float *state = reinterpret_cast<float *>(ws + kAlign);
    const size_t state_bytes = (size_t)B * H * d_k * d_v * 4;
    char *slot0 = ws + kAlign + up(state_bytes);
    struct Slot {
        void *q, *k, *v, *a, *b, *o;
    } slot[2];
    for (int i = 0; i < 2; ++i) {
        char *p = slot0 + i * sp.total();
        slot[i].q = p; p += up(sp.q);
        slot[i].k = p; p += up(sp.k);
        slot[i].v = p; p += up(sp.v);
        slot[i].a = p; p += up(sp.a);
        slot[i].b = p; p += up(sp.b);
        slot[i].o = p;
    }

    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t ev_start = nullptr, ev_end = nullptr, ev_state = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
    kda_status st = KDA_OK;
    auto ok = [&](cudaError_t e) {
        if (e != cudaSuccess && st == KDA_OK) st = KDA_ERR_LAUNCH;
        return st == KDA_OK;
    };
    const unsigned ef = cudaEventDisableTiming;
    if (ok(cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking)) &&
        ok(cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking)) && ok(cudaEventCreateWithFlags(&ev_start, ef)) &&
        ok(cudaEventCreateWithFlags(&ev_end, ef)) && ok(cudaEventCreateWithFlags(&ev_state, ef))) {
        for (int i = 0; i < 2 && st == KDA_OK; ++i)
            ok(cudaEventCreateWithFlags(&ev_in[i], ef)) && ok(cudaEventCreateWithFlags(&ev_done[i], ef)) &&
                ok(cudaEventCreateWithFlags(&ev_out[i], ef));
    }
    // everything below is ordered after the work already queued on the caller's stream
    if (st == KDA_OK && ok(cudaEventRecord(ev_start, stream)) && ok(cudaStreamWaitEvent(h2d, ev_start, 0)) &&
        ok(cudaStreamWaitEvent(d2h, ev_start, 0))) {
        ok(cudaMemsetAsync(status, 0, 16, stream));
        if (initial_state) {
            ok(cudaMemcpyAsync(state, initial_state, state_bytes, cudaMemcpyHostToDevice, h2d)) &&
                ok(cudaEventRecord(ev_state, h2d)) && ok(cudaStreamWaitEvent(stream, ev_state, 0));
        } else {
            ok(cudaMemsetAsync(state, 0, state_bytes, stream));
        }
    }
    const size_t wq = (size_t)d_k * esize(qkv_dtype), wv = (size_t)d_v * esize(qkv_dtype);
    const size_t wa = (size_t)(per_head ? 1 : d_k) * esize(gate_dtype), wb = esize(gate_dtype);
    const size_t wo = (size_t)d_v * esize(out_dtype);
    for (int t0 = 0, j = 0; t0 < T && st == KDA_OK; t0 += S, ++j) {
        const int L = T - t0 < S ? T - t0 : S;
        Slot &sl = slot[j & 1];
        // inputs of segment j into slot j&1, once the kernel of segment j-2 has read it
        if (j >= 2 && !ok(cudaStreamWaitEvent(h2d, ev_done[j & 1], 0))) break;
        for (int b = 0; b < B && st == KDA_OK; ++b) {
            ok(copy_rows(sl.q, q, true, b, T, L, t0, H, wq, h2d)) && ok(copy_rows(sl.k, k, true, b, T, L, t0, H, wq, h2d)) &&
                ok(copy_rows(sl.v, v, true, b, T, L, t0, H, wv, h2d)) &&
                ok(copy_rows(sl.a, alpha, true, b, T, L, t0, H, wa, h2d)) &&
                ok(copy_rows(sl.b, beta, true, b, T, L, t0, H, wb, h2d));
        }
        if (!ok(cudaEventRecord(ev_in[j & 1], h2d)) || !ok(cudaStreamWaitEvent(stream, ev_in[j & 1], 0))) break;
        // the kernel on segment j, continuing from the state in place, once segment j-2's
        // outputs have left slot j&1
        if (j >= 2 && !ok(cudaStreamWaitEvent(stream, ev_out[j & 1], 0))) break;
        const kda_status ks = kda::prefill_launch(kind, sl.q, sl.k, sl.v, sl.a, sl.b, state, sl.o, state, B, L, H,
                                                  d_k, d_v, scale, qkv_dtype, gate_dtype, out_dtype,
                                                  static_cast<unsigned int *>(status), stream);
        if (ks != KDA_OK) {
            st = ks;
            break;
        }
        // outputs of segment j back to the host
        if (!ok(cudaEventRecord(ev_done[j & 1], stream)) || !ok(cudaStreamWaitEvent(d2h, ev_done[j & 1], 0))) break;
        for (int b = 0; b < B && st == KDA_OK; ++b) ok(copy_rows(sl.o, o, false, b, T, L, t0, H, wo, d2h));
        ok(cudaEventRecord(ev_out[j & 1], d2h));
    }
    if (st == KDA_OK && final_state) {
        ok(cudaEventRecord(ev_state, stream)) && ok(cudaStreamWaitEvent(d2h, ev_state, 0)) &&
            ok(cudaMemcpyAsync(final_state, state, state_bytes, cudaMemcpyDeviceToHost, d2h));
    }
    // the caller's stream resumes once every copy back has landed
    if (st == KDA_OK) ok(cudaEventRecord(ev_end, d2h)) && ok(cudaStreamWaitEvent(stream, ev_end, 0));
    // streams and events are released once their queued work has completed
    for (int i = 0; i < 2; ++i) {
        if (ev_in[i]) cudaEventDestroy(ev_in[i]);
        if (ev_done[i]) cudaEventDestroy(ev_done[i]);
        if (ev_out[i]) cudaEventDestroy(ev_out[i]);
    }
    if (ev_start) cudaEventDestroy(ev_start);
    if (ev_end) cudaEventDestroy(ev_end);
    if (ev_state) cudaEventDestroy(ev_state);
    if (h2d) cudaStreamDestroy(h2d);
    if (d2h) cudaStreamDestroy(d2h);
    return st;
}

size_t kda_decode_step_host_workspace_bytes(int N, int H, int d_k, int d_v, kda_dtype qkv_dtype,
                                            kda_dtype gate_dtype, kda_dtype out_dtype)
{
    if (N < 0 || H < 0 || d_k <= 0 || d_v <= 0) return 0;
    return slot_plan(N, 1, H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype, false).total();
}

kda_status kda_decode_step_host(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                                float *state, void *o, int N, int H, int d_k, int d_v, float scale,
                                kda_dtype qkv_dtype, kda_dtype gate_dtype, kda_dtype out_dtype, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream)
{
    if (N < 0 || H < 0 || d_k <= 0 || d_v <= 0) return KDA_ERR_SHAPE;
    if (!dtype_ok(qkv_dtype) || !dtype_ok(gate_dtype) || !dtype_ok(out_dtype)) return KDA_ERR_DTYPE;
    if (!head_ok(d_k) || !head_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (N * (long long)H == 0) return KDA_OK;
    if (!q || !k || !v || !alpha || !beta || !o || !state) return KDA_ERR_NULL;
    const size_t need = kda_decode_step_host_workspace_bytes(N, H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if ((uintptr_t)workspace % kAlign) return KDA_ERR_ALIGN;
    const SlotPlan sp = slot_plan(N, 1, H, d_k, d_v, qkv_dtype, gate_dtype, out_dtype, false);
    char *p = static_cast<char *>(workspace);
    void *dq = p; p += up(sp.q);
    void *dk = p; p += up(sp.k);
    void *dv = p; p += up(sp.v);
    void *da = p; p += up(sp.a);
    void *db = p; p += up(sp.b);
    void *dout = p;
    if (cudaMemcpyAsync(dq, q, sp.q, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, sp.k, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, sp.v, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(da, alpha, sp.a, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(db, beta, sp.b, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return KDA_ERR_LAUNCH;
    const kda_status ks = kda_decode_step(dq, dk, dv, da, db, state, dout, N, H, d_k, d_v, scale, qkv_dtype,
                                          gate_dtype, out_dtype, stream);
    if (ks != KDA_OK) return ks;
    return cudaMemcpyAsync(o, dout, sp.o, cudaMemcpyDeviceToHost, stream) == cudaSuccess ? KDA_OK : KDA_ERR_LAUNCH;
}

}  // extern "C"
