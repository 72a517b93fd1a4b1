// Chunkwise KDA prefill on the sm_100a tensor cores (tcgen05, TMEM accumulators).
//
// Scope: d_k = d_v = 128, bf16 q/k/v, bf16 alpha/beta, fp32 state and output.
// One block (256 threads) per (sequence, head) walks chunks of C = 32 tokens.
//
// Per chunk, with G[r] = sum_{t<=r} log alpha_t (per key channel), an anchor
// a = G[15] in the middle of the chunk, e_r = exp(G_r - a) and
// gamma_r = exp(G_r) (the pages' in-chunk cumulative decay):
//   [A_kk; A_qk]  = [K*e ; Q*e] (K/e)^T        (tensor cores, M=64 N=32 K=128)
//   A_kk <- strict lower * beta_r,   A_qk <- lower incl. diagonal * scale
//   T'   = (I + A_kk)^-1 Diag(beta)             (forward substitution, fp32)
//   W^T  = (K*gamma)^T T'^T,  U^T = V^T T'^T    (tensor cores)
//   E^T  = U^T - S^T W^T,     O^T = S^T (scale Q*gamma)^T
//   O^T += E^T A_qk^T,        dS^T = E^T (K*gamma_end/gamma)
//   S^T  = S^T Diag(gamma_end) + dS^T           (fp32, registers)
// The serial products are computed transposed so that the 128 value channels
// are the MMA's M dimension and each TMEM lane (and thread) owns one value
// channel j: the state column S[:, j] lives in that thread's registers in fp32.
// The anchor keeps every tensor-core operand inside exp(+-16 tokens of decay),
// so both factors stay in range while their product is the exact pairwise
// decay prod_{t=s+1..r} alpha_t.
//
// Precision: every operand that is not an exact bf16 input is split as
// x = hi + lo (two bf16) and each product accumulates hi*hi + hi*lo + lo*hi in
// fp32, which keeps ~16 significant bits; the fp32 accumulations, the
// triangular solve and the state update are exact fp32.
//
// Algorithm: "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two schedules for
// the same recurrence" (provisional errors, the unit-lower-triangular
// correction solved by substitution, the one-shot state fast-forward, the read
// with the diagonal included, decays as differences of prefix sums of
// log alpha); "From Fast Weight Programmers to KDA" (jonahsamost.bearblog.dev),
// section "Kimi Delta Attention" (the WY/UT factors W and U).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace kda {
namespace tc {

constexpr int C = 32;      // tokens per chunk
constexpr int D = 128;     // d_k = d_v
constexpr int NT = 256;    // threads per block
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait

// ---- operand layouts (no swizzle; core matrices of 8 rows x 16 B) ------------
// An (MN x K) bf16 operand is stored as MN/8 x K/8 core matrices; the core
// matrix (mn/8, k/8) sits at (mn/8)*SBO + (k/8)*128 with SBO = (K/8)*128.
// K-major: a core-matrix row is one mn index holding 8 consecutive k.
// MN-major: a core-matrix row is one k index holding 8 consecutive mn.
__device__ __forceinline__ uint32_t kmaj(int mn, int k, int K)
{
    return (uint32_t)((mn >> 3) * (K / 8) * 128 + (k >> 3) * 128 + (mn & 7) * 16 + (k & 7) * 2);
}
__device__ __forceinline__ uint32_t mnmaj(int mn, int k, int K)
{
    return (uint32_t)((mn >> 3) * (K / 8) * 128 + (k >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

// ---- shared-memory plan (bytes) ----------------------------------------------
constexpr int ROWB = 272;                       // staged input row: 256 B + 16 B pad
constexpr int OFF_Q = 0;                        // staged q  [C][ROWB]
constexpr int OFF_K = OFF_Q + C * ROWB;         // staged k
constexpr int OFF_A = OFF_K + C * ROWB;         // staged alpha (bf16)
constexpr int OFF_V0 = OFF_A + C * ROWB;        // V buffers: A operand of U (MN-major, M=j, K=s)
constexpr int OFF_V1 = OFF_V0 + D * C * 2;
constexpr int GROW = D * 4 + 16;                // G row: 128 fp32 + pad
constexpr int OFF_G = OFF_V1 + D * C * 2;       // G [C][GROW]
constexpr int OFF_CST = OFF_G + C * GROW;       // aexp[128], cend[128], gend[128], beta[32]
constexpr int OFF_X = OFF_CST + (3 * D + C) * 4;
//   region X, first use (until the A-products complete):
constexpr int X_LQ_HI = 0;                      // [K*e ; Q*e]  (M=64, K=128, K-major)
constexpr int X_LQ_LO = X_LQ_HI + 64 * D * 2;
constexpr int X_R_HI = X_LQ_LO + 64 * D * 2;    // K/e          (N=32, K=128, K-major)
constexpr int X_R_LO = X_R_HI + C * D * 2;
constexpr int X_BYTES = X_R_LO + C * D * 2;     // 48 KB
//   region X, second use:
constexpr int X_KG_HI = 0;                      // K*gamma  (A of W^T: M=d, K=s, MN-major)
constexpr int X_KG_LO = X_KG_HI + D * C * 2;
constexpr int X_W_HI = X_KG_LO + D * C * 2;     // W        (B of E:   N=r, K=d, MN-major)
constexpr int X_W_LO = X_W_HI + C * D * 2;
constexpr int X_E_HI = X_W_LO + C * D * 2;      // E^T      (A of O/dS: M=j, K=s, K-major)
constexpr int X_E_LO = X_E_HI + D * C * 2;
constexpr int OFF_QG = OFF_X + X_BYTES;         // scale*Q*gamma (B of O: N=r, K=d, K-major) hi, lo
constexpr int OFF_KE = OFF_QG + 2 * C * D * 2;  // K*gamma_end/gamma (B of dS: N=d, K=s, MN-major) hi, lo
constexpr int OFF_TP = OFF_KE + 2 * C * D * 2;  // T' (B of W/U: N=r, K=s, MN-major) hi, lo
constexpr int OFF_AQ = OFF_TP + 2 * C * C * 2;  // A_qk (B of O: N=r, K=s, K-major) hi, lo
constexpr int OFF_AKK = OFF_AQ + 2 * C * C * 2; // A_kk fp32 [C][C+1]
constexpr int OFF_ST = OFF_AKK + C * (C + 1) * 4;   // S^T (A of E/O: M=j, K=d, K-major) hi, lo
constexpr int OFF_BAR = OFF_ST + 2 * D * D * 2;     // 4 mbarriers
constexpr int OFF_MISC = OFF_BAR + 4 * 8;           // tmem base, error flag
constexpr int SMEM_BYTES = OFF_MISC + 16;

// TMEM columns
constexpr uint32_t TM_A = 0, TM_W = 32, TM_E = 64, TM_O = 96, TM_S = 128, TM_COLS = 256;

__device__ __forceinline__ void split2(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Store 8 values as hi and lo bf16 16-byte chunks.
__device__ __forceinline__ void st_split8(uint8_t *hi_base, uint8_t *lo_base, uint32_t off,
                                          const float (&x)[8])
{
    union {
        uint4 u;
        __nv_bfloat16 b[8];
    } h, l;
#pragma unroll
    for (int i = 0; i < 8; ++i) split2(x[i], h.b[i], l.b[i]);
    *reinterpret_cast<uint4 *>(hi_base + off) = h.u;
    *reinterpret_cast<uint4 *>(lo_base + off) = l.u;
}

__device__ __forceinline__ void ld_bf16x8(const uint8_t *p, float (&x)[8])
{
    union {
        uint4 u;
        __nv_bfloat16 b[8];
    } v;
    v.u = *reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = __bfloat162float(v.b[i]);
}

struct Bars {
    uint32_t a, w, e, s;
};

// Issue the cp.async copies of chunk c's q, k, alpha rows (staged) and v (into
// the MN-major V buffer) and load its beta into a register.
__device__ __forceinline__ void prefetch_chunk(const ChunkArgs &p, uint8_t *sm, int b, int h, int t0,
                                               int L, uint32_t v_off, float &beta_reg, int tid)
{
    const size_t HD = (size_t)p.H * D;
    // 32 rows x 16 chunks of 16 B per tensor; 2 chunks per thread per tensor
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int idx = tid + it * NT;      // 0..511
        const int r = idx >> 4, ch = idx & 15;
        const int rr = r < L ? r : 0;
        const uint32_t nbytes = r < L ? 16u : 0u;
        const size_t g = ((size_t)b * p.T + t0 + rr) * HD + (size_t)h * D + ch * 8;
        const uint32_t so = (uint32_t)(r * ROWB + ch * 16);
        ptx::cp_async16(ptx::smem_u32(sm + OFF_Q + so), (const __nv_bfloat16 *)p.q + g, nbytes);
        ptx::cp_async16(ptx::smem_u32(sm + OFF_K + so), (const __nv_bfloat16 *)p.k + g, nbytes);
        ptx::cp_async16(ptx::smem_u32(sm + OFF_A + so), (const __nv_bfloat16 *)p.alpha + g, nbytes);
        // v row r, value channels 8ch..8ch+7 -> MN-major (M = j, K = s = r)
        ptx::cp_async16(ptx::smem_u32(sm + v_off + mnmaj(ch * 8, r, C)), (const __nv_bfloat16 *)p.v + g,
                        nbytes);
    }
    ptx::cp_async_commit();
    if (tid < C) {
        beta_reg = 0.f;
        if (tid < L)
            beta_reg = __bfloat162float(((const __nv_bfloat16 *)p.beta)[((size_t)b * p.T + t0 + tid) * p.H + h]);
    }
}

__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(ChunkArgs p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;

    float *G = reinterpret_cast<float *>(sm + OFF_G);
    float *aexp = reinterpret_cast<float *>(sm + OFF_CST);
    float *cend = aexp + D;
    float *gend = cend + D;
    float *sbeta = gend + D;
    float *Akk = reinterpret_cast<float *>(sm + OFF_AKK);
    uint8_t *X = sm + OFF_X;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *err_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const uint32_t bar0 = ptx::smem_u32(sm + OFF_BAR);
    const Bars bars{bar0, bar0 + 8, bar0 + 16, bar0 + 24};

    if (tid == 0) {
        ptx::mbar_init(bars.a, 1);
        ptx::mbar_init(bars.w, 1);
        ptx::mbar_init(bars.e, 1);
        ptx::mbar_init(bars.s, 1);
        ptx::fence_mbar_init();
        *err_flag = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;   // this warp's TMEM lane quadrant

    // ---- initial state: thread owns value channel j, key channels [64*half, +64)
    const int j = quad * 32 + lane;
    float Sreg[64];
    {
        const size_t tile = (size_t)bh * D * D;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const int d = 64 * half + i;
            Sreg[i] = p.s_in ? p.s_in[tile + (size_t)d * D + j] : 0.f;
        }
        uint8_t *st_hi = sm + OFF_ST, *st_lo = st_hi + D * D * 2;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = Sreg[kb * 8 + i];
            st_split8(st_hi, st_lo, kmaj(j, 64 * half + kb * 8, D), x);
        }
    }

    const int nchunks = (p.T + C - 1) / C;
    float beta_reg = 0.f;
    prefetch_chunk(p, sm, b, h, 0, min(C, p.T), OFF_V0, beta_reg, tid);

    const uint32_t id_A = ptx::idesc_bf16(64, C, 0, 0, 0);
    const uint32_t id_W = ptx::idesc_bf16(128, C, 1, 1, 0);
    const uint32_t id_Eneg = ptx::idesc_bf16(128, C, 0, 1, 1);
    const uint32_t id_O = ptx::idesc_bf16(128, C, 0, 0, 0);
    const uint32_t id_dS = ptx::idesc_bf16(128, D, 0, 1, 0);

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * C;
        const int L = min(C, p.T - t0);
        const uint32_t par = (uint32_t)(c & 1);
        const uint32_t v_off = (c & 1) ? OFF_V1 : OFF_V0;

        // ---- S0: this chunk's inputs have landed
        ptx::cp_async_wait_all();
        if (tid < C) sbeta[tid] = beta_reg;
        __syncthreads();

        // ---- P0: cumulative log-decay per key channel and per-channel constants
        if (tid < D) {
            const int d = tid;
            const __nv_bfloat16 *arow = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_A);
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                const float al = __bfloat162float(arow[r * (ROWB / 2) + d]);
                run += (r < L) ? log_alpha(al) : 0.f;
                G[r * (GROW / 4) + d] = run;
            }
            const float a = G[15 * (GROW / 4) + d];
            aexp[d] = __expf(a);
            cend[d] = __expf(run - a);
            gend[d] = __expf(run);
        }
        __syncthreads();

        // ---- P1: decay-scaled operands of the A-products, Q*gamma and K_end
        {
            const int r = tid & 31;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int g = (tid >> 5) + 8 * it;          // channel group: d = 8g .. 8g+7
                float q8[8], k8[8], e[8], re[8];
                ld_bf16x8(sm + OFF_Q + r * ROWB + g * 16, q8);
                ld_bf16x8(sm + OFF_K + r * ROWB + g * 16, k8);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int d = 8 * g + i;
                    const float x = G[r * (GROW / 4) + d] - G[15 * (GROW / 4) + d];
                    e[i] = __expf(fminf(fmaxf(x, -87.f), 87.f));
                    re[i] = __expf(fminf(fmaxf(-x, -87.f), 87.f));
                }
                float lk[8], lq[8], rk[8], qg[8], ke[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int d = 8 * g + i;
                    lk[i] = k8[i] * e[i];
                    lq[i] = q8[i] * e[i];
                    rk[i] = k8[i] * re[i];
                    qg[i] = p.scale * q8[i] * (e[i] * aexp[d]);
                    ke[i] = rk[i] * cend[d];
                }
                st_split8(X + X_LQ_HI, X + X_LQ_LO, kmaj(r, 8 * g, D), lk);
                st_split8(X + X_LQ_HI, X + X_LQ_LO, kmaj(C + r, 8 * g, D), lq);
                st_split8(X + X_R_HI, X + X_R_LO, kmaj(r, 8 * g, D), rk);
                st_split8(sm + OFF_QG, sm + OFF_QG + C * D * 2, kmaj(r, 8 * g, D), qg);
                st_split8(sm + OFF_KE, sm + OFF_KE + C * D * 2, mnmaj(8 * g, r, C), ke);
            }
        }
        ptx::fence_proxy_async_smem();
        __syncthreads();

        // ---- M1: [K*e; Q*e] (K/e)^T
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t lq[2] = {ptx::smem_u32(X + X_LQ_HI), ptx::smem_u32(X + X_LQ_LO)};
            const uint32_t rr[2] = {ptx::smem_u32(X + X_R_HI), ptx::smem_u32(X + X_R_LO)};
            const int pa[3] = {0, 0, 1}, pb[3] = {0, 1, 0};
            uint32_t acc = 0;
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < D / 16; ++ks) {
                    ptx::mma_bf16(tmem + TM_A, ptx::smem_desc(lq[pa[sp]] + ks * 256, 128, (D / 8) * 128),
                                  ptx::smem_desc(rr[pb[sp]] + ks * 256, 128, (D / 8) * 128), id_A, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.a);
        }

        // ---- P2: A_kk / A_qk from TMEM; K*gamma; the triangular solve
        if (!ptx::mbar_wait(bars.a, par, kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        if (warp < 4) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + TM_A, v);
            ptx::tmem_wait_ld();
            if (lane < 16) {
                const int row = 16 * quad + lane;   // M=64 accumulator rows live in lanes 0-15 of each quadrant
                if (row < C) {
                    const int r = row;
                    const float br = sbeta[r];
#pragma unroll
                    for (int s = 0; s < C; ++s) Akk[r * (C + 1) + s] = (s < r) ? br * v[s] : 0.f;
                } else {
                    const int r = row - C;
#pragma unroll
                    for (int sb = 0; sb < 4; ++sb) {
                        float x[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int s = 8 * sb + i;
                            x[i] = (s <= r) ? p.scale * v[s] : 0.f;
                        }
                        st_split8(sm + OFF_AQ, sm + OFF_AQ + C * C * 2, kmaj(r, 8 * sb, C), x);
                    }
                }
            }
        } else {
            // K*gamma, A operand of W^T (MN-major: M = d, K = s)
            const int t2 = tid - 128;
            const int r = t2 & 31;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int g = (t2 >> 5) + 4 * it;
                float k8[8], kg[8];
                ld_bf16x8(sm + OFF_K + r * ROWB + g * 16, k8);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    kg[i] = k8[i] * __expf(fmaxf(G[r * (GROW / 4) + 8 * g + i], -87.f));
                st_split8(X + X_KG_HI, X + X_KG_LO, mnmaj(8 * g, r, C), kg);
            }
        }
        ptx::tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            // column c = lane of T = (I + A_kk)^-1, then T' = T Diag(beta)
            const int cc = lane;
            float t[C];
#pragma unroll
            for (int i = 0; i < C; ++i) {
                float acc = (i == cc) ? 1.f : 0.f;
#pragma unroll
                for (int jj = 0; jj < i; ++jj) acc = fmaf(-Akk[i * (C + 1) + jj], t[jj], acc);
                t[i] = acc;
            }
            const float bc = sbeta[cc];
#pragma unroll
            for (int ib = 0; ib < 4; ++ib) {
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = t[8 * ib + i] * bc;
                // T' element (r = 8ib+i, s = cc): MN-major (N = r, K = s)
                st_split8(sm + OFF_TP, sm + OFF_TP + C * C * 2, mnmaj(8 * ib, cc, C), x);
            }
        }
        ptx::fence_proxy_async_smem();
        __syncthreads();

        // ---- M2: W^T = (K*gamma)^T T'^T, U^T = V^T T'^T
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t kg[2] = {ptx::smem_u32(X + X_KG_HI), ptx::smem_u32(X + X_KG_LO)};
            const uint32_t tp[2] = {ptx::smem_u32(sm + OFF_TP), ptx::smem_u32(sm + OFF_TP + C * C * 2)};
            const uint32_t vv = ptx::smem_u32(sm + v_off);
            const int pa[3] = {0, 0, 1}, pb[3] = {0, 1, 0};
            uint32_t acc = 0;
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < C / 16; ++ks) {
                    ptx::mma_bf16(tmem + TM_W, ptx::smem_desc(kg[pa[sp]] + ks * 256, 128, (C / 8) * 128),
                                  ptx::smem_desc(tp[pb[sp]] + ks * 256, 128, (C / 8) * 128), id_W, acc);
                    acc = 1;
                }
            acc = 0;
            for (int sp = 0; sp < 2; ++sp)
                for (int ks = 0; ks < C / 16; ++ks) {
                    ptx::mma_bf16(tmem + TM_E, ptx::smem_desc(vv + ks * 256, 128, (C / 8) * 128),
                                  ptx::smem_desc(tp[sp] + ks * 256, 128, (C / 8) * 128), id_W, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.w);
        }

        // ---- P3: W from TMEM into the B operand of E (MN-major: N = r, K = d)
        if (!ptx::mbar_wait(bars.w, par, kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + TM_W + 16 * half, v);
            ptx::tmem_wait_ld();
            const int d = j;   // lane quadrant = key channel for W^T
#pragma unroll
            for (int rb = 0; rb < 2; ++rb) {
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = v[8 * rb + i];
                st_split8(X + X_W_HI, X + X_W_LO, mnmaj(16 * half + 8 * rb, d, D), x);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // staged q/k/alpha are no longer needed: fetch the next chunk now
        if (c + 1 < nchunks) {
            const int t0n = t0 + C;
            prefetch_chunk(p, sm, b, h, t0n, min(C, p.T - t0n), (c & 1) ? OFF_V0 : OFF_V1, beta_reg, tid);
        }

        // ---- M3: E^T -= S^T W^T, O^T = S^T (scale Q gamma)^T
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t st[2] = {ptx::smem_u32(sm + OFF_ST), ptx::smem_u32(sm + OFF_ST + D * D * 2)};
            const uint32_t w[2] = {ptx::smem_u32(X + X_W_HI), ptx::smem_u32(X + X_W_LO)};
            const uint32_t qg[2] = {ptx::smem_u32(sm + OFF_QG), ptx::smem_u32(sm + OFF_QG + C * D * 2)};
            const int pa[3] = {0, 0, 1}, pb[3] = {0, 1, 0};
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < D / 16; ++ks)
                    ptx::mma_bf16(tmem + TM_E, ptx::smem_desc(st[pa[sp]] + ks * 256, 128, (D / 8) * 128),
                                  ptx::smem_desc(w[pb[sp]] + ks * 256, 128, (D / 8) * 128), id_Eneg, 1);
            uint32_t acc = 0;
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < D / 16; ++ks) {
                    ptx::mma_bf16(tmem + TM_O, ptx::smem_desc(st[pa[sp]] + ks * 256, 128, (D / 8) * 128),
                                  ptx::smem_desc(qg[pb[sp]] + ks * 256, 128, (D / 8) * 128), id_O, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.e);
        }

        // ---- C1: E^T from TMEM into the A operand of O and dS (K-major: M = j, K = s)
        if (!ptx::mbar_wait(bars.e, par, kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + TM_E + 16 * half, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int sb = 0; sb < 2; ++sb) {
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = v[8 * sb + i];
                st_split8(X + X_E_HI, X + X_E_LO, kmaj(j, 16 * half + 8 * sb, C), x);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- M4: O^T += E^T A_qk^T, dS^T = E^T K_end
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t et[2] = {ptx::smem_u32(X + X_E_HI), ptx::smem_u32(X + X_E_LO)};
            const uint32_t aq[2] = {ptx::smem_u32(sm + OFF_AQ), ptx::smem_u32(sm + OFF_AQ + C * C * 2)};
            const uint32_t ke[2] = {ptx::smem_u32(sm + OFF_KE), ptx::smem_u32(sm + OFF_KE + C * D * 2)};
            const int pa[3] = {0, 0, 1}, pb[3] = {0, 1, 0};
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < C / 16; ++ks)
                    ptx::mma_bf16(tmem + TM_O, ptx::smem_desc(et[pa[sp]] + ks * 256, 128, (C / 8) * 128),
                                  ptx::smem_desc(aq[pb[sp]] + ks * 256, 128, (C / 8) * 128), id_O, 1);
            uint32_t acc = 0;
            for (int sp = 0; sp < 3; ++sp)
                for (int ks = 0; ks < C / 16; ++ks) {
                    ptx::mma_bf16(tmem + TM_S, ptx::smem_desc(et[pa[sp]] + ks * 256, 128, (C / 8) * 128),
                                  ptx::smem_desc(ke[pb[sp]] + ks * 256, 128, (C / 8) * 128), id_dS, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.s);
        }

        // ---- C2: state update in registers, S^T back to the operand; outputs
        if (!ptx::mbar_wait(bars.s, par, kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            uint8_t *st_hi = sm + OFF_ST, *st_lo = st_hi + D * D * 2;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
                ptx::tmem_ld32(tmem + lane_base + TM_S + 64 * half + 32 * part, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int ii = 32 * part + i;
                    Sreg[ii] = fmaf(gend[64 * half + ii], Sreg[ii], v[i]);
                }
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    float x[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[i] = Sreg[32 * part + 8 * kb + i];
                    st_split8(st_hi, st_lo, kmaj(j, 64 * half + 32 * part + 8 * kb, D), x);
                }
            }
            float o16[16];
            ptx::tmem_ld16(tmem + lane_base + TM_O + 16 * half, o16);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * half + i;
                if (r < L) {
                    const size_t row = ((size_t)b * p.T + t0 + r) * p.H + h;
                    st_elem(p.o, row * D + j, o16[i], p.out_bf16);
                }
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (*err_flag) break;
    }

    if (p.s_out) {
        const size_t tile = (size_t)bh * D * D;
#pragma unroll
        for (int i = 0; i < 64; ++i) p.s_out[tile + (size_t)(64 * half + i) * D + j] = Sreg[i];
    }
    if (*err_flag && tid == 0 && p.status) atomicOr(p.status, 1u);
    ptx::cp_async_wait_all();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace tc

bool chunk_tc_supported(int dk, int dv, kda_dtype qkv, kda_dtype gate)
{
    return dk == tc::D && dv == tc::D && qkv == KDA_BF16 && gate == KDA_BF16;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, int dk, int dv, cudaStream_t stream)
{
    (void)dk; (void)dv;
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(tc::kda_chunk_tc_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    tc::kda_chunk_tc_kernel<<<(unsigned)blocks, tc::NT, tc::SMEM_BYTES, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
