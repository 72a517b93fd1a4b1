// Token-by-token KDA prefill spread over the value columns ("column scan"), for
// workloads with few (sequence, head) pairs.
//
// The chunk kernels walk the chunks of a sequence one after another, so a workload with
// few (sequence, head) pairs is bound by the latency of one chunk step, not by memory or
// arithmetic.  Here every value column of the state is a chain of its own: column j of
// S evolves with the token's k, q, alpha, beta and its own v_j only -- S~ = Diag(alpha) S
// scales each column separately, v^_j = S~[:, j] . k and the write adds k e_j to column j.
// A group of G lanes owns NJ columns, each lane DK/G key channels of them in registers.
// Per token and column, with x = alpha * S[:, j] (this lane's channels):
//   r = k . x,  p = q . x,  k . q              (G-lane sums: log2 G shuffle steps)
//   e = beta (v_j - r),  o_j = scale (p + e (k . q)),  S[:, j] <- x + k e
// (o_t = S_t^T scale q with S_t = S~ + k e^T).  A warp issues its columns' work one
// instruction at a time, so the time of a token is about the warp's instruction count
// for it: few columns and few channels per lane (G = 16, NJ = 1) when the workload has
// SMs to spare, more of both (G = 8, NJ = 2: the token's k, q, alpha and k . q shared by
// two chains) when it has not.  A block of NW warps (1 or 2) owns NW * (32/G) * NJ
// columns of one (sequence, head); the rows of 32 tokens at a time are staged in shared
// memory by cp.async (two stages) and their outputs leave as one tile.
// Recurrence: "Module 03 -- KDA I: The Delta-Rule Recurrence", section 2; schedule:
// "Kimi Delta Attention (KDA)", "Two schedules for the same recurrence" (the fused
// recurrent form, here with the value columns as the parallel dimension).
#pragma once

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace scan {

constexpr int TB = 32;   // tokens per staged tile

// Shared-memory layout for a block owning jb value columns: two stages of raw
// rows {q, k, alpha (per channel), v columns, fp32 scalars beta and alpha (per head)},
// then the o tile [TB][jb] fp32.  Every offset is a multiple of 16 bytes.
struct Layout {
    int q_bytes, a_bytes, v_bytes;
    int off_k, off_a, off_v, off_sc, stage, off_o, bytes;
    __host__ __device__ Layout(int dk, int qs, int gs, bool head_gate, int jb)
    {
        q_bytes = TB * dk * qs;
        a_bytes = head_gate ? 0 : TB * dk * gs;
        v_bytes = (TB * jb * qs + 15) / 16 * 16;
        off_k = q_bytes;
        off_a = 2 * q_bytes;
        off_v = off_a + a_bytes;
        off_sc = off_v + v_bytes;
        stage = off_sc + 2 * TB * 4;
        off_o = 2 * stage;
        bytes = off_o + TB * jb * 4;
    }
};

__device__ __forceinline__ void cp16(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp4(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Channels d and d+1 (d even) of a staged row, widened to fp32.
template <bool kBf16>
__device__ __forceinline__ float2 ld_pair(const uint8_t *row, int d)
{
    if constexpr (kBf16) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + 2 * d);
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    } else {
        return *reinterpret_cast<const float2 *>(row + 4 * d);
    }
}

template <bool kBf16>
__device__ __forceinline__ float ld_one(const uint8_t *p, int idx)
{
    if constexpr (kBf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[idx]);
    else
        return reinterpret_cast<const float *>(p)[idx];
}

// cp.async copies of tile n's q, k, alpha rows and the block's v columns into stage st
// (rows past the sequence's end are neither copied nor read).
template <int DK, bool kQBf16, bool kGBf16, bool kHeadGate>
__device__ __forceinline__ void stage_rows(const ChunkArgs &a, uint8_t *st, const Layout &L, const SeqSpan &sp,
                                           int h, int j0, int jb, int dv, int n, int tid, int nt)
{
    constexpr int QS = kQBf16 ? 2 : 4, GS = kGBf16 ? 2 : 4;
    constexpr int QG = DK * QS / 16, AG = DK * GS / 16;
    const int VG = jb * QS / 4;   // 4-byte pieces of a row's v columns (jb is even)
    const int rows = min(TB, sp.len - n * TB);
    for (int i = tid; i < rows * QG; i += nt) {
        const int r = i / QG, g = i % QG;
        const size_t row = (sp.tok0 + (size_t)n * TB + r) * a.H + h;
        cp16(st + r * DK * QS + 16 * g, (const uint8_t *)a.q + row * DK * QS + 16 * g);
        cp16(st + L.off_k + r * DK * QS + 16 * g, (const uint8_t *)a.k + row * DK * QS + 16 * g);
    }
    if constexpr (!kHeadGate)
        for (int i = tid; i < rows * AG; i += nt) {
            const int r = i / AG, g = i % AG;
            const size_t row = (sp.tok0 + (size_t)n * TB + r) * a.H + h;
            cp16(st + L.off_a + r * DK * GS + 16 * g, (const uint8_t *)a.alpha + row * DK * GS + 16 * g);
        }
    for (int i = tid; i < rows * VG; i += nt) {
        const int r = i / VG, g = i % VG;
        const size_t row = (sp.tok0 + (size_t)n * TB + r) * a.H + h;
        cp4(st + L.off_v + r * jb * QS + 4 * g, (const uint8_t *)a.v + (row * dv + j0) * QS + 4 * g);
    }
}

// beta and the per-head alpha of token n*TB + tid (threads 0..TB-1), loaded into
// registers now and written to the stage later.
template <bool kGBf16, bool kHeadGate>
__device__ __forceinline__ float2 load_scalars(const ChunkArgs &a, const SeqSpan &sp, int h, int n, int tid)
{
    const int t = n * TB + tid;
    if (tid >= TB || t >= sp.len) return make_float2(0.f, 0.f);
    const size_t row = (sp.tok0 + (size_t)t) * a.H + h;
    return make_float2(ld_elem(a.beta, row, kGBf16), kHeadGate ? ld_elem(a.alpha, row, kGBf16) : 1.f);
}

__device__ __forceinline__ void put_scalars(uint8_t *st, const Layout &L, int tid, float2 x)
{
    if (tid < TB) {
        float *sc = reinterpret_cast<float *>(st + L.off_sc);
        sc[tid] = x.x;
        sc[TB + tid] = x.y;
    }
}

// This lane's key channels: d = 2 l + 2 G i + {0, 1} (pairs, one 4- or 8-byte load each)
// when DK is a multiple of 2 G, else d = l + G i.
template <int DK, int G>
struct Chan {
    static constexpr bool kPairs = DK % (2 * G) == 0;
    static constexpr int CPL = DK / G;
    __device__ static constexpr int d(int l, int i) { return kPairs ? 2 * l + 2 * G * (i >> 1) + (i & 1) : l + G * i; }
};

// One token's inputs as this lane reads them: k, q, alpha of its key channels, beta and
// v of its columns.
template <int CPL, int NJ>
struct Tok {
    float k[CPL], q[CPL], al[CPL];
    float beta, v[NJ];
};

template <int DK, int G, int NJ, bool kQBf16, bool kGBf16, bool kHeadGate>
__device__ __forceinline__ void load_token(const uint8_t *st, const Layout &L, int l, int jl, int jstep, int jb,
                                           int r, Tok<DK / G, NJ> &t)
{
    using Ch = Chan<DK, G>;
    constexpr int QS = kQBf16 ? 2 : 4, GS = kGBf16 ? 2 : 4;
    const float *sc = reinterpret_cast<const float *>(st + L.off_sc);
    const uint8_t *qr = st + r * DK * QS, *kr = st + L.off_k + r * DK * QS, *ar = st + L.off_a + r * DK * GS;
    const float ah = kHeadGate ? sc[TB + r] : 1.f;
    if constexpr (Ch::kPairs) {
#pragma unroll
        for (int i = 0; i < Ch::CPL; i += 2) {
            const int d = Ch::d(l, i);
            const float2 kk = ld_pair<kQBf16>(kr, d), qq = ld_pair<kQBf16>(qr, d);
            t.k[i] = kk.x;
            t.k[i + 1] = kk.y;
            t.q[i] = qq.x;
            t.q[i + 1] = qq.y;
            if constexpr (kHeadGate) {
                t.al[i] = ah;
                t.al[i + 1] = ah;
            } else {
                const float2 aa = ld_pair<kGBf16>(ar, d);
                t.al[i] = aa.x;
                t.al[i + 1] = aa.y;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < Ch::CPL; ++i) {
            const int d = Ch::d(l, i);
            t.k[i] = ld_one<kQBf16>(kr, d);
            t.q[i] = ld_one<kQBf16>(qr, d);
            t.al[i] = kHeadGate ? ah : ld_one<kGBf16>(ar, d);
        }
    }
    t.beta = sc[r];
#pragma unroll
    for (int c = 0; c < NJ; ++c) t.v[c] = ld_one<kQBf16>(st + L.off_v, r * jb + jl + c * jstep);
}

// One token on this lane's part of the group's NJ columns (states s[c]): the reads of
// the decayed states and k . q (summed over the group in a fixed order, so that a token's
// result does not depend on where a call starts), the errors, the outputs (written by the
// group's lane 0 into the tile row o) and the writes.
template <int CPL, int G, int NJ>
__device__ __forceinline__ void token_step(const Tok<CPL, NJ> &t, float (&s)[NJ][CPL], float scale, int l,
                                           float *o, int jl, int jstep)
{
    float x[NJ][CPL];
    // two partial sums per dot product (even and odd channels) keep the chains short
    float r[NJ][2], p[NJ][2], kqp[2] = {0.f, 0.f};
#pragma unroll
    for (int c = 0; c < NJ; ++c) r[c][0] = r[c][1] = p[c][0] = p[c][1] = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
            x[c][i] = t.al[i] * s[c][i];
            r[c][i & 1] = fmaf(t.k[i], x[c][i], r[c][i & 1]);
            p[c][i & 1] = fmaf(t.q[i], x[c][i], p[c][i & 1]);
        }
        kqp[i & 1] = fmaf(t.k[i], t.q[i], kqp[i & 1]);
    }
    float rr[NJ], pp[NJ], kq = kqp[0] + kqp[1];
#pragma unroll
    for (int c = 0; c < NJ; ++c) {
        rr[c] = r[c][0] + r[c][1];
        pp[c] = p[c][0] + p[c][1];
    }
#pragma unroll
    for (int off = 1; off < G; off <<= 1) {
#pragma unroll
        for (int c = 0; c < NJ; ++c) {
            rr[c] += __shfl_xor_sync(0xffffffffu, rr[c], off);
            pp[c] += __shfl_xor_sync(0xffffffffu, pp[c], off);
        }
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
#pragma unroll
    for (int c = 0; c < NJ; ++c) {
        const float e = t.beta * (t.v[c] - rr[c]);
        if (l == 0) o[jl + c * jstep] = scale * fmaf(e, kq, pp[c]);
#pragma unroll
        for (int i = 0; i < CPL; ++i) s[c][i] = fmaf(t.k[i], e, x[c][i]);
    }
}

template <int DK, int G, int NJ, bool kQBf16, bool kGBf16, bool kHeadGate>
__global__ void __launch_bounds__(64) kda_scan_kernel(const ChunkArgs a, int dv)
{
    constexpr int CPL = DK / G;        // key channels per lane
    constexpr int GPW = 32 / G;        // column groups per warp
    extern __shared__ __align__(16) uint8_t sm[];
    const int nt = blockDim.x, nw = nt >> 5;
    const int jstep = GPW * nw, jb = jstep * NJ;   // columns of the block; group's column stride
    const Layout L(DK, kQBf16 ? 2 : 4, kGBf16 ? 2 : 4, kHeadGate, jb);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane / G, l = lane % G;
    const int ncb = dv / jb;
    const int cb = blockIdx.x % ncb, bh = blockIdx.x / ncb;
    const int b = bh / a.H, h = bh % a.H;
    // the group's columns: j0 + jl + c * jstep, c < NJ
    const int j0 = cb * jb, jl = GPW * warp + g;
    SeqSpan sp;
    if (!sequence_span(a, b, sp)) {
        if (tid == 0 && a.status) atomicOr(a.status, 2u);
        return;
    }
    const size_t tile = (size_t)bh * DK * dv;

    float s[NJ][CPL];   // S[d][column c] for this lane's channels d
#pragma unroll
    for (int c = 0; c < NJ; ++c)
#pragma unroll
        for (int i = 0; i < CPL; ++i)
            s[c][i] = a.s_in ? a.s_in[tile + (size_t)Chan<DK, G>::d(l, i) * dv + j0 + jl + c * jstep] : 0.f;

    const int ntiles = (sp.len + TB - 1) / TB;
    float *osm = reinterpret_cast<float *>(sm + L.off_o);
    if (ntiles > 0) {
        stage_rows<DK, kQBf16, kGBf16, kHeadGate>(a, sm, L, sp, h, j0, jb, dv, 0, tid, nt);
        put_scalars(sm, L, tid, load_scalars<kGBf16, kHeadGate>(a, sp, h, 0, tid));
    }
    cp_commit();
    for (int n = 0; n < ntiles; ++n) {
        uint8_t *st = sm + (n & 1) * L.stage;
        uint8_t *nx = sm + ((n + 1) & 1) * L.stage;
        float2 xn = make_float2(0.f, 0.f);
        if (n + 1 < ntiles) {
            stage_rows<DK, kQBf16, kGBf16, kHeadGate>(a, nx, L, sp, h, j0, jb, dv, n + 1, tid, nt);
            xn = load_scalars<kGBf16, kHeadGate>(a, sp, h, n + 1, tid);
        }
        cp_commit();
        cp_wait_one();     // this thread's copies of tile n have landed
        __syncthreads();   // and every thread's
        const int rows = min(TB, sp.len - n * TB);
        // two tokens per pass: the second token's rows are read before the first token's
        // serial part, so the shared-memory loads are not on the chain
#pragma unroll 1
        for (int r = 0; r < rows; r += 2) {
            Tok<CPL, NJ> t0, t1;
            load_token<DK, G, NJ, kQBf16, kGBf16, kHeadGate>(st, L, l, jl, jstep, jb, r, t0);
            const bool two = r + 1 < rows;
            if (two) load_token<DK, G, NJ, kQBf16, kGBf16, kHeadGate>(st, L, l, jl, jstep, jb, r + 1, t1);
            token_step<CPL, G, NJ>(t0, s, a.scale, l, osm + r * jb, jl, jstep);
            if (two) token_step<CPL, G, NJ>(t1, s, a.scale, l, osm + (r + 1) * jb, jl, jstep);
        }
        put_scalars(nx, L, tid, xn);
        __syncthreads();   // the o tile is complete; stage n is no longer read
        for (int i = tid; i < rows * jb; i += nt) {
            const int r = i / jb, c = i % jb;
            const size_t row = (sp.tok0 + (size_t)n * TB + r) * a.H + h;
            st_elem(a.o, row * dv + j0 + c, osm[i], a.out_bf16);
        }
    }
    if (a.s_out) {
#pragma unroll
        for (int c = 0; c < NJ; ++c)
#pragma unroll
            for (int i = 0; i < CPL; ++i)
                a.s_out[tile + (size_t)Chan<DK, G>::d(l, i) * dv + j0 + jl + c * jstep] = s[c][i];
    }
}

// The current device's SM count (148 on a B200), looked up once per device.
inline int device_sms()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int DK, int G, int NJ>
cudaError_t launch_scan_shape(const ChunkArgs &a, int dv, int nw, cudaStream_t stream)
{
    const int jb = nw * (32 / G) * NJ;
    const long long blocks = (long long)a.B * a.H * (dv / jb);
    auto pick = [&](auto kernel, bool qb, bool gb, bool hg) -> cudaError_t {
        const int bytes = Layout(DK, qb ? 2 : 4, gb ? 2 : 4, hg, jb).bytes;
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (err != cudaSuccess) return err;
        kernel<<<(unsigned)blocks, 32 * nw, bytes, stream>>>(a, dv);
        return cudaGetLastError();
    };
#define KDA_SCAN_CASE(QB, GB, HG)                                              \
    if (a.qkv_bf16 == QB && a.gate_bf16 == GB && (a.gate_per_head != 0) == HG) \
        return pick(kda_scan_kernel<DK, G, NJ, QB, GB, HG>, QB, GB, HG);
    KDA_SCAN_CASE(true, true, false)
    KDA_SCAN_CASE(true, false, false)
    KDA_SCAN_CASE(false, true, false)
    KDA_SCAN_CASE(false, false, false)
    KDA_SCAN_CASE(true, true, true)
    KDA_SCAN_CASE(true, false, true)
    KDA_SCAN_CASE(false, true, true)
    KDA_SCAN_CASE(false, false, true)
#undef KDA_SCAN_CASE
    return cudaErrorInvalidValue;
}

// Latency form (one column a group, one warp a block; G = 16 lanes a column from d_k = 64
// up, 8 below, where 16 would leave a lane one or two channels) while its warps fit on
// the SMs at kLatencyWarpsPerSm a piece; otherwise the throughput form (G = 8, NJ = 2:
// 8 columns a warp, two warps a block when there are at least two a SM).  Measured on a
// B200 at T = 2048: 4 heads, d = 64: 0.37 ms latency form against 0.49 ms throughput
// form; 1184 heads: 4.4 against 5.2 ms for the 8-lane one-column form.
template <int DK>
cudaError_t launch_scan_dk(const ChunkArgs &a, int dv, cudaStream_t stream)
{
    constexpr long long kLatencyWarpsPerSm = 4;
    constexpr int kLatencyLanes = DK >= 64 ? 16 : 8;
    const long long pairs = (long long)a.B * a.H;
    if (pairs == 0) return cudaSuccess;
    const int sms = device_sms();
    if (pairs * dv / (32 / kLatencyLanes) <= kLatencyWarpsPerSm * sms)
        return launch_scan_shape<DK, kLatencyLanes, 1>(a, dv, 1, stream);
    return launch_scan_shape<DK, 8, 2>(a, dv, pairs * dv / 8 >= 2LL * sms ? 2 : 1, stream);
}

}  // namespace scan
}  // namespace kda
