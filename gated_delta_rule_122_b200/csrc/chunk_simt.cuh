// Chunkwise KDA on CUDA cores, fp32 throughout: the general path for every
// supported head size and input dtype (the tensor-core kernel covers
// d_k = d_v = 128 with bf16 q/k/v).
//
// One block per (sequence, head); chunks of C = 32 tokens are walked in order
// with the state S [DK x DV] resident in shared memory.  For a chunk with
// cumulative log-decay G[r] = sum_{t<=r} log alpha_t (per key channel):
//   Akk[r][s] = beta_r sum_d k_rd k_sd exp(G_rd - G_sd)           s <  r
//   Aqk[r][s] =        sum_d q_rd k_sd exp(G_rd - G_sd)           s <= r
//   (I + Akk) W = Diag(beta) (K * exp(G)),  (I + Akk) U = Diag(beta) V
//   E = U - W S                          (the true in-chunk errors)
//   O = scale ((Q * exp(G)) S + Aqk E)
//   S <- Diag(exp(G_end)) S + (K * exp(G_end - G))^T E
// Every pairwise decay exp(G_r - G_s), s <= r, is formed directly, so no
// factor ever exceeds 1 and no anchoring is needed on this path.
// GDN-2 ("From Fast Weight Programmers to KDA", section "Gated DeltaNet-2"):
// with an erase gate b_r (per key channel) and a write gate w_r (per value
// channel) instead of beta_r, the same steps run with
//   Akk[r][s] = sum_d b_rd k_rd k_sd exp(G_rd - G_sd),
//   (I + Akk) W = (b * K) * exp(G),   (I + Akk) U = w * V.
// With raw inputs the staging applies the preprocessing first: q_r and k_r divided
// by their L2 norms, G from log alpha = -softplus(gate logit), beta = sigmoid(logit).
// Algorithm: "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two schedules for
// the same recurrence"; "From Fast Weight Programmers to KDA"
// (jonahsamost.bearblog.dev), section "Kimi Delta Attention".
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace kda {


constexpr int kSimtChunk = 32;
constexpr int kSimtChunkRows = kSimtChunk;
// Threads per block: DV value columns x NRG row groups, with the most row groups
// (up to 32) that keep the block within 512 threads and divide both the chunk and
// DK (16 warps per SM hide the shared-memory latency of the fp32 loops better than 8).
template <int DK, int DV>
constexpr int simt_row_groups()
{
    int g = 32;
    while (g > 1 && (DV * g > 512 || kSimtChunkRows % g != 0 || DK % g != 0)) g /= 2;
    return g;
}
template <int DK, int DV>
constexpr int simt_threads()
{
    return DV * simt_row_groups<DK, DV>();
}

template <int DK, int DV>
struct SimtLayout {
    static constexpr int C = kSimtChunk;
    static constexpr int PK = DK + 1, PV = DV + 1, PC = C + 1;
    static constexpr int oQ = 0;
    static constexpr int oK = oQ + C * PK;
    static constexpr int oG = oK + C * PK;
    static constexpr int oW = oG + C * PK;
    static constexpr int oV = oW + C * PK;
    static constexpr int oE = oV + C * PV;
    static constexpr int oS = oE + C * PV;
    static constexpr int PT = C + 4;              // row pitch of A_kk^T (16-byte rows)
    static constexpr int oAkk = oS + DK * DV;     // A_kk^T: column s of A_kk as row s
    static constexpr int oAqk = oAkk + C * PT;
    static constexpr int oBeta = oAqk + C * PC;
    static constexpr int oNrm = oBeta + C;      // 1/||q_r||, 1/||k_r|| (raw inputs)
    static constexpr int floats = oNrm + 2 * C;
    static constexpr size_t bytes = sizeof(float) * (size_t)floats;
};

template <int DK, int DV, bool kGdn2>
__global__ void __launch_bounds__(simt_threads<DK, DV>())
kda_chunk_simt_kernel(ChunkArgs a)
{
    using Ly = SimtLayout<DK, DV>;
    constexpr int C = Ly::C, PK = Ly::PK, PV = Ly::PV, PC = Ly::PC, NT = simt_threads<DK, DV>();
    constexpr int NRG = NT / DV;          // row groups for value-column loops
    constexpr int RPT_C = C / NRG;        // chunk rows per thread
    constexpr int RPT_K = DK / NRG;       // key rows per thread (state update)
    static_assert(NT % DV == 0 && C % NRG == 0 && DK % NRG == 0, "thread mapping");

    extern __shared__ float sm[];
    float *Q = sm + Ly::oQ, *K = sm + Ly::oK, *G = sm + Ly::oG, *W = sm + Ly::oW;
    float *V = sm + Ly::oV, *E = sm + Ly::oE, *S = sm + Ly::oS;
    float *Akk = sm + Ly::oAkk, *Aqk = sm + Ly::oAqk, *Bt = sm + Ly::oBeta, *Nrm = sm + Ly::oNrm;

    const int bh = blockIdx.x;                 // sequence * H + head (state tile)
    const int h = bh % a.H;
    const int tid = threadIdx.x;
    const size_t tile = (size_t)bh * DK * DV;
    SeqSpan sp;                                // the sequence's token rows
    if (!sequence_span(a, bh / a.H, sp)) {
        if (tid == 0 && a.status) atomicOr(a.status, 2u);
        return;
    }

    for (int idx = tid; idx < DK * DV; idx += NT)
        S[idx] = a.s_in ? a.s_in[tile + idx] : 0.f;

    const int jcol = tid % DV, rgrp = tid / DV;

    for (int t0 = 0; t0 < sp.len; t0 += C) {
        const int L = min(C, sp.len - t0);
        // 1. stage the chunk; rows >= L are identity steps (k = q = v = 0, alpha = 1, beta = 0)
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int r = idx / DK, d = idx % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (r < L) {
                const size_t row = (sp.tok0 + t0 + r) * a.H + h;
                qv = ld_elem(a.q, row * DK + d, a.qkv_bf16);
                kv = ld_elem(a.k, row * DK + d, a.qkv_bf16);
                const float x = ld_elem(a.alpha, a.gate_per_head ? row : row * DK + d, a.gate_bf16);
                gv = a.raw_inputs ? log_alpha_from_logit(x) : log_alpha(x);
            }
            Q[r * PK + d] = qv; K[r * PK + d] = kv; G[r * PK + d] = gv;
            if constexpr (kGdn2) {   // the erase-gated key b * k, the left factor of Akk
                const size_t row = (sp.tok0 + t0 + r) * a.H + h;
                W[r * PK + d] = (r < L) ? ld_elem(a.erase, row * DK + d, a.gate_bf16) * kv : 0.f;
            }
        }
        for (int idx = tid; idx < C * DV; idx += NT) {
            const int r = idx / DV, j = idx % DV;
            float vv = 0.f;
            if (r < L) {
                const size_t row = (sp.tok0 + t0 + r) * a.H + h;
                vv = ld_elem(a.v, row * DV + j, a.qkv_bf16);
            }
            V[r * PV + j] = vv;
        }
        if constexpr (!kGdn2) {   // GDN-2 has no beta tensor
            for (int r = tid; r < C; r += NT) {
                const float y = (r < L) ? ld_elem(a.beta, (sp.tok0 + t0 + r) * a.H + h, a.gate_bf16) : 0.f;
                Bt[r] = (r < L) ? (a.raw_inputs ? sigmoid_of(y) : y) : 0.f;
            }
        }
        __syncthreads();
        if (a.raw_inputs) {   // q_r / ||q_r||, k_r / ||k_r||
            for (int r = tid; r < 2 * C; r += NT) {
                const float *x = (r < C) ? Q + r * PK : K + (r - C) * PK;
                float ss = 0.f;
                for (int d = 0; d < DK; ++d) ss = fmaf(x[d], x[d], ss);
                Nrm[r] = inv_norm(ss);
            }
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += NT) {
                const int r = idx / DK, d = idx % DK;
                Q[r * PK + d] *= Nrm[r];
                K[r * PK + d] *= Nrm[C + r];
            }
            __syncthreads();
        }

        // 2. inclusive cumulative log-decay per key channel
        for (int d = tid; d < DK; d += NT) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) { run += G[r * PK + d]; G[r * PK + d] = run; }
        }
        __syncthreads();

        // 3. interaction matrices and the right-hand sides of the triangular solves
        for (int p = tid; p < C * C; p += NT) {
            const int r = p / C, s = p % C;
            float akk = 0.f, aqk = 0.f;
            if (s <= r) {
                for (int d = 0; d < DK; ++d) {
                    const float ks = K[s * PK + d] * __expf(G[r * PK + d] - G[s * PK + d]);
                    akk = fmaf(kGdn2 ? W[r * PK + d] : K[r * PK + d], ks, akk);
                    aqk = fmaf(Q[r * PK + d], ks, aqk);
                }
            }
            Akk[s * Ly::PT + r] = (s < r) ? (kGdn2 ? akk : Bt[r] * akk) : 0.f;
            Aqk[r * PC + s] = aqk;
        }
        if constexpr (kGdn2) __syncthreads();   // the Akk loop above read W
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int r = idx / DK, d = idx % DK;
            if constexpr (kGdn2) W[r * PK + d] *= __expf(G[r * PK + d]);
            else W[r * PK + d] = Bt[r] * K[r * PK + d] * __expf(G[r * PK + d]);
        }
        for (int idx = tid; idx < C * DV; idx += NT) {
            const int r = idx / DV, j = idx % DV;
            if constexpr (kGdn2) {
                const size_t row = (sp.tok0 + t0 + r) * a.H + h;
                V[r * PV + j] *= (r < L) ? ld_elem(a.wgate, row * DV + j, a.gate_bf16) : 0.f;
            } else {
                V[r * PV + j] *= Bt[r];
            }
        }
        __syncthreads();

        // 4. forward substitution (I + Akk) X = RHS, one column per thread, right-looking:
        //    once x_j is final it is subtracted from every later row, so the 31 updates of
        //    a step are independent and column j of A_kk is read as 16-byte vectors (row j
        //    of the transposed copy); then the decay-scaled operands of the inter-chunk
        //    products
        for (int col = tid; col < DK + DV; col += NT) {
            float *X = (col < DK) ? (W + col) : (V + (col - DK));
            const int stride = (col < DK) ? PK : PV;
            float x[C];
#pragma unroll
            for (int i = 0; i < C; ++i) x[i] = X[i * stride];
#pragma unroll
            for (int j = 0; j < C - 1; ++j) {
                const float xj = x[j];
#pragma unroll
                for (int i4 = (j + 1) / 4; i4 < C / 4; ++i4) {
                    const float4 a = *reinterpret_cast<const float4 *>(Akk + j * Ly::PT + 4 * i4);
                    if (4 * i4 + 0 > j) x[4 * i4 + 0] = fmaf(-a.x, xj, x[4 * i4 + 0]);
                    if (4 * i4 + 1 > j) x[4 * i4 + 1] = fmaf(-a.y, xj, x[4 * i4 + 1]);
                    if (4 * i4 + 2 > j) x[4 * i4 + 2] = fmaf(-a.z, xj, x[4 * i4 + 2]);
                    if (4 * i4 + 3 > j) x[4 * i4 + 3] = fmaf(-a.w, xj, x[4 * i4 + 3]);
                }
            }
#pragma unroll
            for (int i = 0; i < C; ++i) X[i * stride] = x[i];
        }
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int r = idx / DK, d = idx % DK;
            const float g = G[r * PK + d];
            Q[r * PK + d] *= __expf(g);                            // q * gamma_r
            K[r * PK + d] *= __expf(G[(C - 1) * PK + d] - g);      // k * gamma_end / gamma_r
        }
        __syncthreads();

        // 5. E = U - W S and the inter-chunk read (Q * gamma) S: each S element is read
        //    once per thread and used for all of the thread's rows
        float oacc[RPT_C], eacc[RPT_C];
#pragma unroll
        for (int m = 0; m < RPT_C; ++m) {
            eacc[m] = V[(rgrp + NRG * m) * PV + jcol];
            oacc[m] = 0.f;
        }
        for (int d = 0; d < DK; ++d) {
            const float sdj = S[d * DV + jcol];
#pragma unroll
            for (int m = 0; m < RPT_C; ++m) {
                const int r = rgrp + NRG * m;
                eacc[m] = fmaf(-W[r * PK + d], sdj, eacc[m]);
                oacc[m] = fmaf(Q[r * PK + d], sdj, oacc[m]);
            }
        }
#pragma unroll
        for (int m = 0; m < RPT_C; ++m) E[(rgrp + NRG * m) * PV + jcol] = eacc[m];
        __syncthreads();

        // 6. outputs: O = scale (inter + Aqk E)
#pragma unroll
        for (int m = 0; m < RPT_C; ++m) {
            const int r = rgrp + NRG * m;
            float o = oacc[m];
            for (int s = 0; s <= r; ++s) o = fmaf(Aqk[r * PC + s], E[s * PV + jcol], o);
            if (r < L) {
                const size_t row = (sp.tok0 + t0 + r) * a.H + h;
                st_elem(a.o, row * DV + jcol, a.scale * o, a.out_bf16);
            }
        }
        // 7. state fast-forward: S <- Diag(gamma_end) S + K_end^T E, eight state rows at a
        //    time so that each E element read serves eight of them
        constexpr int SG = (RPT_K % 8 == 0) ? 8 : 1;
        for (int m0 = 0; m0 < RPT_K; m0 += SG) {
            float acc[SG];
#pragma unroll
            for (int g = 0; g < SG; ++g) {
                const int i = rgrp + NRG * (m0 + g);
                acc[g] = S[i * DV + jcol] * __expf(G[(C - 1) * PK + i]);
            }
            for (int r = 0; r < C; ++r) {
                const float erj = E[r * PV + jcol];
#pragma unroll
                for (int g = 0; g < SG; ++g) acc[g] = fmaf(K[r * PK + rgrp + NRG * (m0 + g)], erj, acc[g]);
            }
#pragma unroll
            for (int g = 0; g < SG; ++g) S[(rgrp + NRG * (m0 + g)) * DV + jcol] = acc[g];
        }
        __syncthreads();
    }

    if (a.s_out)
        for (int idx = tid; idx < DK * DV; idx += NT) a.s_out[tile + idx] = S[idx];
}

template <int DK, int DV>
static cudaError_t launch_chunk_simt_t(const ChunkArgs &a, cudaStream_t stream)
{
    using Ly = SimtLayout<DK, DV>;
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    auto kernel = a.erase ? kda_chunk_simt_kernel<DK, DV, true> : kda_chunk_simt_kernel<DK, DV, false>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly::bytes);
    if (err != cudaSuccess) return err;
    kernel<<<(unsigned)blocks, simt_threads<DK, DV>(), Ly::bytes, stream>>>(a);
    return cudaGetLastError();
}

// Launch for one key size DK and any supported value size (instantiated per DK in the
// chunk_simt_dk*.cu files, which compile in parallel).
template <int DK>
cudaError_t launch_chunk_simt_dk(const ChunkArgs &a, int dv, cudaStream_t s)
{
    switch (dv) {
    case 16: return launch_chunk_simt_t<DK, 16>(a, s);
    case 32: return launch_chunk_simt_t<DK, 32>(a, s);
    case 48: return launch_chunk_simt_t<DK, 48>(a, s);
    case 64: return launch_chunk_simt_t<DK, 64>(a, s);
    case 80: return launch_chunk_simt_t<DK, 80>(a, s);
    case 96: return launch_chunk_simt_t<DK, 96>(a, s);
    case 112: return launch_chunk_simt_t<DK, 112>(a, s);
    case 128: return launch_chunk_simt_t<DK, 128>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
