// Token-by-token KDA prefill spread over the value columns ("column scan"), for
// workloads with few (sequence, head) pairs.
//
// The chunk kernels walk the chunks of a sequence one after another, so a workload with
// few (sequence, head) pairs is bound by the latency of one chunk step, not by memory or
// arithmetic.  Here every value column of the state is a chain of its own: column j of
// S evolves with the token's k, q, alpha, beta and its own v_j only -- S~ = Diag(alpha) S
// scales each column separately, v^_j = S~[:, j] . k and the write adds k e_j to column j.
// One group of 8 lanes owns column j, each lane DK/8 key channels in registers (channel
// pairs d = 2 l + 16 i + {0, 1} for lane l of the group).  Per token, with x = alpha * S[:, j]
// (this lane's channels):
//   r = k . x,  p = q . x,  k . q              (8-lane sums: three shuffle steps)
//   e = beta (v_j - r),  o_j = scale (p + e (k . q)),  S[:, j] <- x + k e
// (o_t = S_t^T scale q with S_t = S~ + k e^T), so the serial path of a token is a
// DK/16-step dot product, three shuffle steps and two multiply-adds.  A block of NW warps
// (1, 2 or 4, chosen at launch) owns 4 NW value columns of one (sequence, head); the
// rows of 32 tokens at a time are staged in shared memory by cp.async (two stages) and
// their outputs leave as one tile.
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

// Shared-memory layout for a block of nw warps (4 nw value columns): two stages of raw
// rows {q, k, alpha (per channel), v columns, fp32 scalars beta and alpha (per head)},
// then the o tile [TB][4 nw] fp32.  Every offset is a multiple of 16 bytes.
struct Layout {
    int q_bytes, a_bytes, v_bytes;
    int off_k, off_a, off_v, off_sc, stage, off_o, bytes;
    __host__ __device__ Layout(int dk, int qs, int gs, bool head_gate, int nw)
    {
        q_bytes = TB * dk * qs;
        a_bytes = head_gate ? 0 : TB * dk * gs;
        v_bytes = (TB * 4 * nw * qs + 15) / 16 * 16;
        off_k = q_bytes;
        off_a = 2 * q_bytes;
        off_v = off_a + a_bytes;
        off_sc = off_v + v_bytes;
        stage = off_sc + 2 * TB * 4;
        off_o = 2 * stage;
        bytes = off_o + TB * 4 * nw * 4;
    }
};

__device__ __forceinline__ void cp16(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp8(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem) : "memory");
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
    const int VG = jb * QS / 8;   // 8-byte pieces of a row's v columns
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
        cp8(st + L.off_v + r * jb * QS + 8 * g, (const uint8_t *)a.v + (row * dv + j0) * QS + 8 * g);
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

// One token's inputs as this lane reads them: k, q, alpha of its key channels, beta and
// v of its column.
template <int CPL>
struct Tok {
    float k[CPL], q[CPL], al[CPL];
    float beta, v;
};

template <int DK, bool kQBf16, bool kGBf16, bool kHeadGate>
__device__ __forceinline__ void load_token(const uint8_t *st, const Layout &L, int l, int jl, int jb, int r,
                                           Tok<DK / 8> &t)
{
    constexpr int QS = kQBf16 ? 2 : 4, GS = kGBf16 ? 2 : 4;
    const float *sc = reinterpret_cast<const float *>(st + L.off_sc);
    const uint8_t *qr = st + r * DK * QS, *kr = st + L.off_k + r * DK * QS, *ar = st + L.off_a + r * DK * GS;
    const float ah = kHeadGate ? sc[TB + r] : 1.f;
#pragma unroll
    for (int i = 0; i < DK / 16; ++i) {
        const int d = 2 * l + 16 * i;
        const float2 kk = ld_pair<kQBf16>(kr, d), qq = ld_pair<kQBf16>(qr, d);
        t.k[2 * i] = kk.x;
        t.k[2 * i + 1] = kk.y;
        t.q[2 * i] = qq.x;
        t.q[2 * i + 1] = qq.y;
        if constexpr (kHeadGate) {
            t.al[2 * i] = ah;
            t.al[2 * i + 1] = ah;
        } else {
            const float2 aa = ld_pair<kGBf16>(ar, d);
            t.al[2 * i] = aa.x;
            t.al[2 * i + 1] = aa.y;
        }
    }
    t.beta = sc[r];
    t.v = ld_one<kQBf16>(st + L.off_v, r * jb + jl);
}

// One token on this lane's part of column j (the state s): the two reads of the decayed
// state and k . q (summed over the group in a fixed order, so that a token's result does
// not depend on where a call starts), the error, the output (written by the group's
// lane 0) and the write.
template <int CPL>
__device__ __forceinline__ void token_step(const Tok<CPL> &t, float (&s)[CPL], float scale, int l, float *o)
{
    float x[CPL];
    float r0 = 0.f, r1 = 0.f, p0 = 0.f, p1 = 0.f, kq0 = 0.f, kq1 = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; i += 2) {
        x[i] = t.al[i] * s[i];
        x[i + 1] = t.al[i + 1] * s[i + 1];
        r0 = fmaf(t.k[i], x[i], r0);
        p0 = fmaf(t.q[i], x[i], p0);
        r1 = fmaf(t.k[i + 1], x[i + 1], r1);
        p1 = fmaf(t.q[i + 1], x[i + 1], p1);
        kq0 = fmaf(t.k[i], t.q[i], kq0);
        kq1 = fmaf(t.k[i + 1], t.q[i + 1], kq1);
    }
    float rr = r0 + r1, pp = p0 + p1, kq = kq0 + kq1;
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
        rr += __shfl_xor_sync(0xffffffffu, rr, off);
        pp += __shfl_xor_sync(0xffffffffu, pp, off);
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
    const float e = t.beta * (t.v - rr);
    if (l == 0) *o = scale * fmaf(e, kq, pp);
#pragma unroll
    for (int i = 0; i < CPL; ++i) s[i] = fmaf(t.k[i], e, x[i]);
}

template <int DK, bool kQBf16, bool kGBf16, bool kHeadGate>
__global__ void __launch_bounds__(128) kda_scan_kernel(const ChunkArgs a, int dv)
{
    constexpr int CPL = DK / 8;   // key channels per lane
    extern __shared__ __align__(16) uint8_t sm[];
    const int nt = blockDim.x, nw = nt >> 5, jb = 4 * nw;
    const Layout L(DK, kQBf16 ? 2 : 4, kGBf16 ? 2 : 4, kHeadGate, nw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 3, l = lane & 7;
    const int ncb = dv / jb;
    const int cb = blockIdx.x % ncb, bh = blockIdx.x / ncb;
    const int b = bh / a.H, h = bh % a.H;
    const int j0 = cb * jb, jl = 4 * warp + g, j = j0 + jl;
    SeqSpan sp;
    if (!sequence_span(a, b, sp)) {
        if (tid == 0 && a.status) atomicOr(a.status, 2u);
        return;
    }
    const size_t tile = (size_t)bh * DK * dv;

    float s[CPL];   // S[d][j] for this lane's channels d = 2 l + 16 i + {0, 1}
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int d = 2 * l + 16 * (i >> 1) + (i & 1);
        s[i] = a.s_in ? a.s_in[tile + (size_t)d * dv + j] : 0.f;
    }

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
            Tok<CPL> t0, t1;
            load_token<DK, kQBf16, kGBf16, kHeadGate>(st, L, l, jl, jb, r, t0);
            const bool two = r + 1 < rows;
            if (two) load_token<DK, kQBf16, kGBf16, kHeadGate>(st, L, l, jl, jb, r + 1, t1);
            token_step<CPL>(t0, s, a.scale, l, osm + r * jb + jl);
            if (two) token_step<CPL>(t1, s, a.scale, l, osm + (r + 1) * jb + jl);
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
        for (int i = 0; i < CPL; ++i) {
            const int d = 2 * l + 16 * (i >> 1) + (i & 1);
            a.s_out[tile + (size_t)d * dv + j] = s[i];
        }
    }
}

// Warps per block: as many as keep at least one block per SM (fewer warps per block
// spread a small workload over more SMs; more share the staged rows).
inline int warps_per_block(long long warps, int sms)
{
    return warps >= 4LL * sms ? 4 : warps >= 2LL * sms ? 2 : 1;
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

template <int DK>
cudaError_t launch_scan_dk(const ChunkArgs &a, int dv, cudaStream_t stream)
{
    const long long warps = (long long)a.B * a.H * dv / 4;   // 4 value columns per warp
    if (warps == 0) return cudaSuccess;
    const int nw = warps_per_block(warps, device_sms());
    const long long blocks = (long long)a.B * a.H * (dv / (4 * nw));
    auto pick = [&](auto kernel, bool qb, bool gb, bool hg) -> cudaError_t {
        const int bytes = Layout(DK, qb ? 2 : 4, gb ? 2 : 4, hg, nw).bytes;
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (err != cudaSuccess) return err;
        kernel<<<(unsigned)blocks, 32 * nw, bytes, stream>>>(a, dv);
        return cudaGetLastError();
    };
#define KDA_SCAN_CASE(QB, GB, HG)                                              \
    if (a.qkv_bf16 == QB && a.gate_bf16 == GB && (a.gate_per_head != 0) == HG) \
        return pick(kda_scan_kernel<DK, QB, GB, HG>, QB, GB, HG);
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

}  // namespace scan
}  // namespace kda
