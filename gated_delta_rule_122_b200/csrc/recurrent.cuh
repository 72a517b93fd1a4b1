// Token-by-token KDA (the "fused recurrent" schedule) and the fused decode step.
//
// One block owns one (sequence, head) state tile S [DK x DV] fp32 in registers.
// Thread t holds float4 column group cg = t % NCG (columns 4cg..4cg+3) of rows
// rg + NRG*m, m < RPT, so every warp-wide load or store of a state row is a
// contiguous, fully coalesced 128-bit access.  Per token:
//   A  stage q, k, alpha, v, beta of the token in shared memory (double buffer)
//   B  one pass over the registers: S <- Diag(alpha) S, and the two partial
//      reductions r = S~^T k and p = S~^T q over this thread's rows
//   C  finish the reductions across row groups; e = beta (v - r);
//      o = scale (p + e (k . q))   [o = S_t^T q with S_t = S~ + k e^T]
//   D  S <- S~ + k e^T in registers
// The decode step is this with T = 1 and the state read from and written back
// to the same buffer; the state is read once and written once.  Multi-token
// decode (the T draft tokens of a speculative step) is this with T > 1 over a
// pool of state slots, optionally storing the state after every token so that
// the step can be rolled back to any accepted prefix.
// Raw inputs: q and k are read un-normalised and their norms, found with k . q,
// scale the two reads and the write; alpha = exp(-softplus(x)), beta = sigmoid(y).
// GDN-2 ("From Fast Weight Programmers to KDA", section "Gated DeltaNet-2"):
// r = S~^T (b * k) with the erase gate b, and e = w * v - r with the write gate w.
// Recurrence: "Module 03 -- KDA I: The Delta-Rule Recurrence", section 2;
// schedule: "Kimi Delta Attention (KDA)", "Two schedules for the same
// recurrence" (fused recurrent).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace kda {

// The largest divisor of n that is at most cap (at least 1).
constexpr int largest_divisor_upto(int n, int cap)
{
    int g = cap < 1 ? 1 : (cap > n ? n : cap);
    while (g > 1 && n % g != 0) --g;
    return g;
}

template <int DK, int DV>
struct RecurrentShape {
    static constexpr int NCG = DV / 4;                                  // float4 column groups
    // row groups: about 256 threads per block, each row group a divisor of DK
    static constexpr int NRG = largest_divisor_upto(DK, 256 / NCG);
    static constexpr int NT = NCG * NRG;                                // threads
    static constexpr int RPT = DK / NRG;                                // rows per thread
    static_assert(NRG * RPT == DK, "rows must split evenly");
};


template <int DK, int DV, bool kGdn2, bool kRaw>
__global__ void __launch_bounds__(RecurrentShape<DK, DV>::NT)
kda_recurrent_kernel(RecurrentArgs a)
{
    using Sh = RecurrentShape<DK, DV>;
    constexpr int NCG = Sh::NCG, NRG = Sh::NRG, RPT = Sh::RPT, NT = Sh::NT;

    // s_e, red_r and red_p are accessed as float4: their alignment is stated, not left to layout
    __shared__ float s_q[2][DK], s_k[2][DK], s_a[2][DK], s_v[2][DV];
    __shared__ __align__(16) float s_e[2][DV];
    __shared__ float s_beta[2], s_kq[2], s_nk[2], s_nq[2];
    __shared__ float s_b[kGdn2 ? 2 : 1][kGdn2 ? DK : 1], s_w[kGdn2 ? 2 : 1][kGdn2 ? DV : 1];
    __shared__ __align__(16) float red_r[NRG][DV];
    __shared__ __align__(16) float red_p[NRG][DV];

    const int bh = blockIdx.x;           // b * H + h
    const int b = bh / a.H, h = bh % a.H;
    const int tid = threadIdx.x;
    const int cg = tid % NCG, rg = tid / NCG;
    int slot = b;
    if (a.state_slots) {   // decode over a slot pool
        slot = a.state_slots[b];
        if (slot < 0) return;
        if (slot >= a.num_slots) {
            if (tid == 0 && a.status) atomicOr(a.status, 2u);
            return;
        }
    }
    const size_t tile = ((size_t)slot * a.H + h) * DK * DV;

    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int i = rg + NRG * m;
        s[m] = a.s_in ? ld_f4_stream(a.s_in + tile + (size_t)i * DV + 4 * cg)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int t = 0; t < a.T; ++t) {
        const int buf = t & 1;
        const size_t row = ((size_t)b * a.T + t) * a.H + h;   // token-head index
        // A: stage the token's vectors
        for (int i = tid; i < DK; i += NT) {
            s_q[buf][i] = ld_elem(a.q, row * DK + i, a.qkv_bf16);
            s_k[buf][i] = ld_elem(a.k, row * DK + i, a.qkv_bf16);
            const float x = ld_elem(a.alpha, a.gate_per_head ? row : row * DK + i, a.gate_bf16);
            s_a[buf][i] = kRaw ? __expf(log_alpha_from_logit(x)) : x;
        }
        for (int j = tid; j < DV; j += NT) s_v[buf][j] = ld_elem(a.v, row * DV + j, a.qkv_bf16);
        if constexpr (kGdn2) {
            for (int i = tid; i < DK; i += NT) s_b[buf][i] = ld_elem(a.erase, row * DK + i, a.gate_bf16);
            for (int j = tid; j < DV; j += NT) s_w[buf][j] = ld_elem(a.wgate, row * DV + j, a.gate_bf16);
        } else {
            if (tid == 0) {
                const float y = ld_elem(a.beta, row, a.gate_bf16);
                s_beta[buf] = kRaw ? sigmoid_of(y) : y;
            }
        }
        __syncthreads();

        // B: decay in registers and the two partial reductions
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int i = rg + NRG * m;
            const float al = s_a[buf][i], qq = s_q[buf][i];
            const float kk = kGdn2 ? s_b[buf][i] * s_k[buf][i] : s_k[buf][i];   // retrieval key
            s[m].x *= al; s[m].y *= al; s[m].z *= al; s[m].w *= al;
            r.x = fmaf(kk, s[m].x, r.x); r.y = fmaf(kk, s[m].y, r.y);
            r.z = fmaf(kk, s[m].z, r.z); r.w = fmaf(kk, s[m].w, r.w);
            p.x = fmaf(qq, s[m].x, p.x); p.y = fmaf(qq, s[m].y, p.y);
            p.z = fmaf(qq, s[m].z, p.z); p.w = fmaf(qq, s[m].w, p.w);
        }
        *reinterpret_cast<float4 *>(&red_r[rg][4 * cg]) = r;
        *reinterpret_cast<float4 *>(&red_p[rg][4 * cg]) = p;
        if (tid < 32) {   // k . q over the key channels (and, for raw inputs, the norms)
            float kq = 0.f, kk = 0.f, qq = 0.f;
            for (int i = tid; i < DK; i += 32) {
                const float ki = s_k[buf][i], qi = s_q[buf][i];
                kq = fmaf(ki, qi, kq);
                if constexpr (kRaw) {
                    kk = fmaf(ki, ki, kk);
                    qq = fmaf(qi, qi, qq);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                kq += __shfl_xor_sync(0xffffffffu, kq, off);
                if constexpr (kRaw) {
                    kk += __shfl_xor_sync(0xffffffffu, kk, off);
                    qq += __shfl_xor_sync(0xffffffffu, qq, off);
                }
            }
            if (tid == 0) {
                const float nk = kRaw ? inv_norm(kk) : 1.f, nq = kRaw ? inv_norm(qq) : 1.f;
                s_kq[buf] = kq * nk * nq;
                s_nk[buf] = nk;
                s_nq[buf] = nq;
            }
        }
        __syncthreads();

        // C: error and output for each value channel
        for (int j = tid; j < DV; j += NT) {
            float rr = 0.f, pp = 0.f;
#pragma unroll
            for (int g = 0; g < NRG; ++g) { rr += red_r[g][j]; pp += red_p[g][j]; }
            if constexpr (kRaw) {   // reads with the unit key and query
                rr *= s_nk[buf];
                pp *= s_nq[buf];
            }
            const float e = kGdn2 ? s_w[buf][j] * s_v[buf][j] - rr : s_beta[buf] * (s_v[buf][j] - rr);
            s_e[buf][j] = e;
            st_elem(a.o, row * DV + j, a.scale * fmaf(e, s_kq[buf], pp), a.out_bf16);
        }
        __syncthreads();

        // D: the rank-one write
        const float4 e4 = *reinterpret_cast<const float4 *>(&s_e[buf][4 * cg]);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const float kk = kRaw ? s_k[buf][rg + NRG * m] * s_nk[buf] : s_k[buf][rg + NRG * m];
            s[m].x = fmaf(kk, e4.x, s[m].x); s[m].y = fmaf(kk, e4.y, s[m].y);
            s[m].z = fmaf(kk, e4.z, s[m].z); s[m].w = fmaf(kk, e4.w, s[m].w);
        }
        if (a.token_states) {   // the state after this token
            float *ts = a.token_states + (((size_t)b * a.T + t) * a.H + h) * DK * DV;
#pragma unroll
            for (int m = 0; m < RPT; ++m) st_f4_stream(ts + (size_t)(rg + NRG * m) * DV + 4 * cg, s[m]);
        }
    }

    if (a.s_out) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int i = rg + NRG * m;
            st_f4_stream(a.s_out + tile + (size_t)i * DV + 4 * cg, s[m]);
        }
    }
}

template <int DK, int DV>
static cudaError_t launch_recurrent_t(const RecurrentArgs &a, cudaStream_t stream)
{
    using Sh = RecurrentShape<DK, DV>;
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (a.erase && a.raw_inputs) return cudaErrorInvalidValue;   // no entry point combines them
    if (a.erase)
        kda_recurrent_kernel<DK, DV, true, false><<<(unsigned)blocks, Sh::NT, 0, stream>>>(a);
    else if (a.raw_inputs)
        kda_recurrent_kernel<DK, DV, false, true><<<(unsigned)blocks, Sh::NT, 0, stream>>>(a);
    else
        kda_recurrent_kernel<DK, DV, false, false><<<(unsigned)blocks, Sh::NT, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_recurrent_dk(const RecurrentArgs &a, int dv, cudaStream_t s)
{
    switch (dv) {
    case 16: return launch_recurrent_t<DK, 16>(a, s);
    case 32: return launch_recurrent_t<DK, 32>(a, s);
    case 48: return launch_recurrent_t<DK, 48>(a, s);
    case 64: return launch_recurrent_t<DK, 64>(a, s);
    case 80: return launch_recurrent_t<DK, 80>(a, s);
    case 96: return launch_recurrent_t<DK, 96>(a, s);
    case 112: return launch_recurrent_t<DK, 112>(a, s);
    case 128: return launch_recurrent_t<DK, 128>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
