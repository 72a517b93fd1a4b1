// Chunkwise KDA prefill on the sm_100a tensor cores (tcgen05, TMEM accumulators).
//
// Scope: d_k = d_v = 128, bf16 q/k/v, bf16 alpha/beta, fp32 state and output.
// One block per (sequence, head) walks chunks of C = 32 tokens: 16 compute warps
// and one warp whose lane 0 issues every tcgen05.mma.
//
// Per chunk, with G[r] = sum_{t<=r} log alpha_t (per key channel), an anchor
// a = G[15] in the middle of the chunk and e_r = exp(G_r - a):
//   Lk = K*e, Lq = scale*Q*e, R = K/e            (bf16 hi/lo operands)
//   [A_kk; A_qk]  = [Lk; Lq] R^T                 (M=64 N=32 K=128)
//   A_kk <- strict lower * beta_r,  A_qk <- lower incl. diagonal
//   T'   = (I + A_kk)^-1 Diag(beta)              (blocked substitution, fp32)
//   W'^T = Lk^T T'^T,   U^T = V^T T'^T           (W' = W Diag(exp(-a)))
//   S'   = Diag(exp(a)) S                        (so that W S = W' S')
//   [O | E]^T = U^T + S'^T [Lq | -W']^T          (S' read from TMEM)
//   O^T += E^T A_qk^T,   dS^T = E^T R
//   S    <- Diag(gamma_end) S + Diag(exp(G_end - a)) dS   (fp32, registers)
// with gamma_r = exp(G_r) the pages' in-chunk cumulative decay
// (scale*Q*gamma = Lq Diag(exp(a)), K*gamma_end/gamma = R Diag(exp(G_end - a))).
// The anchor bounds every operand by exp(16 tokens of decay); products are the
// exact pairwise decays.
//
// Precision: operands that are not exact bf16 inputs are split x = hi + lo.
// Each product runs as two MMAs per K step, A_hi x [B_hi | B_lo] and
// A_lo x [B_hi | B_lo], with the two B planes concatenated along N, so the
// accumulator holds (hi + lo)(hi + lo) in two column groups that are summed
// when read.  Operands are stored "plane-interleaved": each 8-row block keeps
// its hi core matrices followed by its lo core matrices, so one buffer serves
// as a single-plane operand, as a two-plane N-concatenated operand, and
// (swapping the descriptor strides) as the transposed operand.
//
// The serial products are computed transposed: value channel j is the MMA's
// M index and TMEM lane, and compute thread (quad, sub, lane) owns
// S[32sub..32sub+31, j] in fp32 registers.
//
// Schedule: a software pipeline over two chunks.  Compute warps run, per
// iteration c: prep of chunk c+1 | E(c) | A(c+1) readout and solve | state
// update c, S'(c+1), o(c) | W'(c+1); the issuer runs M3(c), M1(c+1), M4(c),
// M2(c+1) as their inputs become ready.  mbarriers carry readiness both ways;
// every wait is bounded.
//
// Algorithm: "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two schedules for
// the same recurrence"; "From Fast Weight Programmers to KDA"
// (jonahsamost.bearblog.dev), section "Kimi Delta Attention".
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace kda {
namespace tc {

constexpr int C = 32;            // tokens per chunk
constexpr int D = 128;           // d_k = d_v
constexpr int NCW = 16;          // compute warps
constexpr int NCT = NCW * 32;    // compute threads
constexpr int NT = NCT + 32;     // + the MMA-issuer warp
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait
constexpr int kComputeBar = 1;   // named barrier id of the compute warps

// ---- plane-interleaved K-major operand layout ------------------------------------
// Row-block (row/8) of an operand with K columns is K*32 bytes: the hi plane's
// K/8 core matrices (128 B each), then the lo plane's.  Element (row, k, plane):
__device__ __forceinline__ uint32_t ipl(int row, int k, int plane, int K)
{
    return (uint32_t)((row >> 3) * (K * 32) + plane * (K * 16) + (k >> 3) * 128 + (row & 7) * 16 +
                      (k & 7) * 2);
}
// Plain MN-major layout (V): core matrices (mn/8, k/8) at (mn/8)*(K/8)*128 + (k/8)*128.
__device__ __forceinline__ uint32_t mnmaj(int mn, int k, int K)
{
    return (uint32_t)((mn >> 3) * (K / 8) * 128 + (k >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

// ---- shared-memory plan (bytes) ----------------------------------------------------
constexpr int ROWB = 272;                              // staged row: 256 B + 16 B pad
constexpr int OFF_STG = 0;                             // staged q, k, alpha of one chunk
constexpr int STG_Q = 0, STG_K = C * ROWB, STG_A = 2 * C * ROWB;
constexpr int OFF_V = OFF_STG + 3 * C * ROWB;          // 2 x V (A of U^T: M=j, K=s, MN-major)
constexpr int V_BYTES = D * C * 2;
constexpr int OFF_CST = OFF_V + 2 * V_BYTES;           // 2 x {aexp, cend, gend}[128] fp32
constexpr int CST_BYTES = 3 * D * 4;
constexpr int OFF_BETA = OFF_CST + 2 * CST_BYTES;      // 2 x beta[32]
constexpr int OFF_LQR = OFF_BETA + 2 * C * 4;          // 2 stages: [Lk; Lq; -W'] rows 0..95, then R
constexpr int LQ_BYTES = 3 * C * D * 4;                // 96 rows x 128 x 2 planes x 2 B
constexpr int R_OFF = LQ_BYTES;
constexpr int LQR_BYTES = LQ_BYTES + C * D * 4;
constexpr int OFF_ET = OFF_LQR + 2 * LQR_BYTES;        // E^T (A of O/dS: rows j, K = s)
constexpr int OFF_TP = OFF_ET + D * C * 4;             // T'  (B of W'/U: rows r, K = s)
constexpr int OFF_AQ = OFF_TP + C * C * 4;             // 2 x A_qk (B of O: rows r, K = s)
constexpr int AQ_BYTES = C * C * 4;
constexpr int OFF_AKK = OFF_AQ + 2 * AQ_BYTES;         // A_kk fp32 [C][C+1]
constexpr int OFF_TS = OFF_AKK + C * (C + 1) * 4;      // T fp32 [C][C+1]
constexpr int OFF_TX = OFF_TS + C * (C + 1) * 4;       // solve temporaries fp32 [3][8][9]
constexpr int OFF_BAR = OFF_TX + 1024;                 // 8 mbarriers
constexpr int OFF_MISC = OFF_BAR + 8 * 8;              // tmem base, error flag
constexpr int SMEM_BYTES = OFF_MISC + 16;

// TMEM columns
constexpr uint32_t TM_A = 0;      // [A_kk; A_qk] (M=64 layout, N=64), then W'^T (N=64)
constexpr uint32_t TM_O = 64;     // O^T (64 cols: hi/lo groups), directly followed by
constexpr uint32_t TM_E = 128;    // E^T (64 cols) so that one N=128 MMA writes both
constexpr uint32_t TM_S = 192;    // dS^T (128 cols)
constexpr uint32_t TM_SP = 320;   // S'^T hi (64 cols) and lo (64 cols), the A operand of M3
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ void split2(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Store 8 values (consecutive k) as hi and lo 16-byte chunks; lo sits plane_gap after hi.
__device__ __forceinline__ void st_split8(uint8_t *p, int plane_gap, const float (&x)[8])
{
    union {
        uint4 u;
        __nv_bfloat16 b[8];
    } h, l;
#pragma unroll
    for (int i = 0; i < 8; ++i) split2(x[i], h.b[i], l.b[i]);
    *reinterpret_cast<uint4 *>(p) = h.u;
    *reinterpret_cast<uint4 *>(p + plane_gap) = l.u;
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

__device__ __forceinline__ void cbar() { ptx::named_bar_sync(kComputeBar, NCT); }

// cp.async copies of chunk n's q, k, alpha rows (staging) and v rows (V buffer
// n&1); 2048 16-byte copies, 4 per compute thread.  Rows past the sequence end
// are zero-filled without reading memory.
__device__ __forceinline__ void prefetch_chunk(const ChunkArgs &p, uint8_t *sm, int b, int h, int n,
                                               int tid)
{
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t HD = (size_t)p.H * D;
    uint8_t *vb = sm + OFF_V + (n & 1) * V_BYTES;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int idx = tid + it * NCT;         // 0..2047; tensor = it
        const int rem = idx & 511;
        const int r = rem >> 4, ch = rem & 15;
        const int rr = r < L ? r : 0;
        const uint32_t nbytes = r < L ? 16u : 0u;
        const size_t g = ((size_t)b * p.T + t0 + rr) * HD + (size_t)h * D + ch * 8;
        if (it == 0)
            ptx::cp_async16(ptx::smem_u32(sm + OFF_STG + STG_Q + r * ROWB + ch * 16),
                            (const __nv_bfloat16 *)p.q + g, nbytes);
        else if (it == 1)
            ptx::cp_async16(ptx::smem_u32(sm + OFF_STG + STG_K + r * ROWB + ch * 16),
                            (const __nv_bfloat16 *)p.k + g, nbytes);
        else if (it == 2)
            ptx::cp_async16(ptx::smem_u32(sm + OFF_STG + STG_A + r * ROWB + ch * 16),
                            (const __nv_bfloat16 *)p.alpha + g, nbytes);
        else   // v row r, value channels 8ch..8ch+7 -> MN-major (M = j, K = s = r)
            ptx::cp_async16(ptx::smem_u32(vb + mnmaj(ch * 8, r, C)), (const __nv_bfloat16 *)p.v + g,
                            nbytes);
    }
    ptx::cp_async_commit();
}

__device__ __forceinline__ float load_beta(const ChunkArgs &p, int b, int h, int n, int r)
{
    const int t = n * C + r;
    if (t >= p.T) return 0.f;
    return __bfloat162float(((const __nv_bfloat16 *)p.beta)[((size_t)b * p.T + t) * p.H + h]);
}

// Signal the issuer: every compute warp arrives once (count NCW).
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane)
{
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}

struct Bars {
    uint32_t a, w, e, s;            // issuer -> compute (tcgen05.commit)
    uint32_t rc, re, rg, rj;        // compute -> issuer (one arrive per compute warp)
};

// ---- the MMA-issuer warp (lane 0) -------------------------------------------------
__device__ void issuer(const ChunkArgs &p, uint8_t *sm, uint32_t tmem, const Bars &bars, int nchunks,
                       volatile int *err_flag)
{
    const uint32_t id_A = ptx::idesc_bf16(64, 64, 0, 0, 0);      // [Lk;Lq] x [R_hi|R_lo]
    const uint32_t id_W = ptx::idesc_bf16(128, 64, 1, 0, 0);     // Lk^T (MN view) x T'
    const uint32_t id_OE = ptx::idesc_bf16(128, 128, 0, 0, 0);   // S' x [Lq | -W']
    const uint32_t id_O2 = ptx::idesc_bf16(128, 64, 0, 0, 0);    // E^T x A_qk
    const uint32_t id_dS = ptx::idesc_bf16(128, 128, 0, 1, 0);   // E^T x R (MN view)
    for (int c = -1; c < nchunks; ++c) {
        const int cn = c + 1;
        if (c >= 0) {   // M3(c): [O | E]^T += S'^T [Lq | -W']^T
            if (!ptx::mbar_wait(bars.rj, (uint32_t)(c & 1), kWaitLimitNs)) { *err_flag = 1; return; }
            ptx::tc_fence_after();
            const uint32_t b0 = ptx::smem_u32(sm + OFF_LQR + (c & 1) * LQR_BYTES) + 4 * D * 32;
            for (int ks = 0; ks < D / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl)
                    ptx::mma_bf16_ts(tmem + TM_O, tmem + TM_SP + 64 * pl + 8 * ks,
                                     ptx::smem_desc(b0 + 256 * ks, 128, D * 16), id_OE, 1);
            ptx::mma_commit(bars.e);
        }
        if (cn < nchunks) {   // M1(cn): [Lk; Lq] x [R_hi | R_lo]^T
            if (!ptx::mbar_wait(bars.rc, (uint32_t)(cn & 1), kWaitLimitNs)) { *err_flag = 1; return; }
            ptx::tc_fence_after();
            const uint32_t lq = ptx::smem_u32(sm + OFF_LQR + (cn & 1) * LQR_BYTES);
            const uint32_t rr = lq + R_OFF;
            uint32_t acc = 0;
            for (int ks = 0; ks < D / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl) {
                    ptx::mma_bf16(tmem + TM_A, ptx::smem_desc(lq + D * 16 * pl + 256 * ks, 128, D * 32),
                                  ptx::smem_desc(rr + 256 * ks, 128, D * 16), id_A, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.a);
        }
        if (c >= 0) {   // M4(c): O^T += E^T A_qk^T, dS^T = E^T R
            if (!ptx::mbar_wait(bars.re, (uint32_t)(c & 1), kWaitLimitNs)) { *err_flag = 1; return; }
            ptx::tc_fence_after();
            const uint32_t et = ptx::smem_u32(sm + OFF_ET);
            const uint32_t aq = ptx::smem_u32(sm + OFF_AQ + (c & 1) * AQ_BYTES);
            const uint32_t rr = ptx::smem_u32(sm + OFF_LQR + (c & 1) * LQR_BYTES) + R_OFF;
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl)
                    ptx::mma_bf16(tmem + TM_O, ptx::smem_desc(et + C * 16 * pl + 256 * ks, 128, C * 32),
                                  ptx::smem_desc(aq + 256 * ks, 128, C * 16), id_O2, 1);
            uint32_t acc = 0;
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pa = 0; pa < 2; ++pa)
                    for (int pb = 0; pb < 2; ++pb) {
                        // R as the MN-major (N = d, K = s) operand: d-blocks 128 B apart,
                        // s-blocks (row-blocks) D*32 B apart
                        ptx::mma_bf16(tmem + TM_S,
                                      ptx::smem_desc(et + C * 16 * pa + 256 * ks, 128, C * 32),
                                      ptx::smem_desc(rr + D * 16 * pb + 2 * D * 32 * ks, D * 32, 128),
                                      id_dS, acc);
                        acc = 1;
                    }
            ptx::mma_commit(bars.s);
        }
        if (cn < nchunks) {   // M2(cn): W'^T = Lk^T T'^T (into TM_A), U^T = V^T T'^T (into TM_E)
            if (!ptx::mbar_wait(bars.rg, (uint32_t)(cn & 1), kWaitLimitNs)) { *err_flag = 1; return; }
            ptx::tc_fence_after();
            const uint32_t lk = ptx::smem_u32(sm + OFF_LQR + (cn & 1) * LQR_BYTES);
            const uint32_t tp = ptx::smem_u32(sm + OFF_TP);
            const uint32_t vv = ptx::smem_u32(sm + OFF_V + (cn & 1) * V_BYTES);
            uint32_t acc = 0;
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl) {
                    // Lk as the MN-major (M = d, K = s) operand
                    ptx::mma_bf16(tmem + TM_A,
                                  ptx::smem_desc(lk + D * 16 * pl + 2 * D * 32 * ks, D * 32, 128),
                                  ptx::smem_desc(tp + 256 * ks, 128, C * 16), id_W, acc);
                    acc = 1;
                }
            for (int ks = 0; ks < C / 16; ++ks)
                ptx::mma_bf16(tmem + TM_E, ptx::smem_desc(vv + 256 * ks, 128, (C / 8) * 128),
                              ptx::smem_desc(tp + 256 * ks, 128, C * 16), id_W, ks > 0);
            ptx::mma_commit(bars.w);
        }
        if (*err_flag) return;
    }
}

// ---- T = (I + A)^-1 for the strictly lower A (fp32, blocks of 8) ---------------------
__device__ void blocked_solve(const float *A, float *T, float *X, int tid)
{
    constexpr int P = C + 1;
    if (tid < 32) {   // diagonal blocks: lane = (block, column)
        const int bk = tid >> 3, cc = tid & 7;
        float t[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float acc = (i == cc) ? 1.f : 0.f;
#pragma unroll
            for (int jj = 0; jj < i; ++jj) acc = fmaf(-A[(8 * bk + i) * P + 8 * bk + jj], t[jj], acc);
            t[i] = acc;
            T[(8 * bk + i) * P + 8 * bk + cc] = acc;
        }
    }
    cbar();
    // T_ij = -T_ii sum_{m=j}^{i-1} A_im T_mj, by distance i-j = 1, 2, 3
#pragma unroll 1
    for (int dist = 1; dist <= 3; ++dist) {
        const int nblk = 4 - dist;
        if (tid < 64 * nblk) {
            const int blk = tid >> 6, pp = (tid >> 3) & 7, qq = tid & 7;
            const int i = blk + dist, j = blk;
            float y = 0.f;
            for (int m = j; m < i; ++m)
#pragma unroll
                for (int k = 0; k < 8; ++k) y = fmaf(A[(8 * i + pp) * P + 8 * m + k], T[(8 * m + k) * P + 8 * j + qq], y);
            X[(blk * 8 + pp) * 9 + qq] = y;
        }
        cbar();
        if (tid < 64 * nblk) {
            const int blk = tid >> 6, pp = (tid >> 3) & 7, qq = tid & 7;
            const int i = blk + dist, j = blk;
            float t = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) t = fmaf(T[(8 * i + pp) * P + 8 * i + k], X[(blk * 8 + k) * 9 + qq], t);
            T[(8 * i + pp) * P + 8 * j + qq] = -t;
        }
        cbar();
    }
}

__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(ChunkArgs p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, sub = (warp >> 2) & 3;
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int nchunks = (p.T + C - 1) / C;

    float *Akk = reinterpret_cast<float *>(sm + OFF_AKK);
    float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
    float *Tx = reinterpret_cast<float *>(sm + OFF_TX);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *err_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const uint32_t bar0 = ptx::smem_u32(sm + OFF_BAR);
    const Bars bars{bar0,      bar0 + 8,  bar0 + 16, bar0 + 24,
                    bar0 + 32, bar0 + 40, bar0 + 48, bar0 + 56};

    if (tid == 0) {
        ptx::mbar_init(bars.a, 1);
        ptx::mbar_init(bars.w, 1);
        ptx::mbar_init(bars.e, 1);
        ptx::mbar_init(bars.s, 1);
        ptx::mbar_init(bars.rc, NCW);
        ptx::mbar_init(bars.re, NCW);
        ptx::mbar_init(bars.rg, NCW);
        ptx::mbar_init(bars.rj, NCW);
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

    if (warp == NCW) {   // the MMA-issuer warp
        if (lane == 0) issuer(p, sm, tmem, bars, nchunks, err_flag);
    } else {
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;   // TMEM lane quadrant
        const int j = quad * 32 + lane;                           // value channel (or key channel d)
        float Sreg[32];
        {
            const size_t tile = (size_t)bh * D * D;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                Sreg[i] = p.s_in ? p.s_in[tile + (size_t)(32 * sub + i) * D + j] : 0.f;
        }
        prefetch_chunk(p, sm, b, h, 0, tid);
        float beta_reg = (tid < C) ? load_beta(p, b, h, 0, tid) : 0.f;
        float *sbeta_all = reinterpret_cast<float *>(sm + OFF_BETA);

        for (int c = -1; c < nchunks; ++c) {
            const int cn = c + 1;
            const bool chain = c >= 0, prep = cn < nchunks;
            uint8_t *lqr_n = sm + OFF_LQR + (cn & 1) * LQR_BYTES;

            // ---- C: prep of chunk cn: prefix sums of log alpha; Lk, Lq, R; constants
            if (prep) {
                if (tid < C) {
                    sbeta_all[(cn & 1) * C + tid] = beta_reg;
                    if (cn + 1 < nchunks) beta_reg = load_beta(p, b, h, cn + 1, tid);
                }
                ptx::cp_async_wait_all();
                cbar();
                const int r = lane, g = warp;     // row r, key channels 8g .. 8g+7
                const int Lc = min(C, p.T - cn * C);
                float q8[8], k8[8], x[8];
                ld_bf16x8(sm + OFF_STG + STG_Q + r * ROWB + g * 16, q8);
                ld_bf16x8(sm + OFF_STG + STG_K + r * ROWB + g * 16, k8);
                ld_bf16x8(sm + OFF_STG + STG_A + r * ROWB + g * 16, x);
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = (r < Lc) ? log_alpha(x[i]) : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float y = __shfl_up_sync(0xffffffffu, x[i], off);
                        if (lane >= off) x[i] += y;
                    }
                }
                float lk[8], lq[8], rk[8];
                float *cst = reinterpret_cast<float *>(sm + OFF_CST + (cn & 1) * CST_BYTES);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a = __shfl_sync(0xffffffffu, x[i], 15);
                    const float gl = __shfl_sync(0xffffffffu, x[i], 31);
                    const float t = x[i] - a;
                    const float e = __expf(fminf(fmaxf(t, -87.f), 87.f));
                    const float re = __expf(fminf(fmaxf(-t, -87.f), 87.f));
                    lk[i] = k8[i] * e;
                    lq[i] = p.scale * q8[i] * e;
                    rk[i] = k8[i] * re;
                    if (lane == 0) {
                        const int d = 8 * g + i;
                        cst[d] = __expf(fmaxf(a, -87.f));                          // exp(a)
                        cst[D + d] = __expf(fminf(fmaxf(gl - a, -87.f), 87.f));    // exp(G_end - a)
                        cst[2 * D + d] = __expf(fmaxf(gl, -87.f));                 // gamma_end
                    }
                }
                st_split8(lqr_n + ipl(r, 8 * g, 0, D), D * 16, lk);
                st_split8(lqr_n + ipl(C + r, 8 * g, 0, D), D * 16, lq);
                st_split8(lqr_n + R_OFF + ipl(r, 8 * g, 0, D), D * 16, rk);
                ptx::fence_proxy_async_smem();
                warp_arrive(bars.rc, lane);
                cbar();   // staging consumed by every warp: fetch the next chunk into it
                if (cn + 1 < nchunks) prefetch_chunk(p, sm, b, h, cn + 1, tid);
            }

            // ---- E: E^T(c) = U^T + (S'^T)(-W')^T from TMEM into the A operand of O/dS
            if (chain) {
                if (!ptx::mbar_wait(bars.e, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
                ptx::tc_fence_after();
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + TM_E + 16 * sub, v);
                ptx::tmem_wait_ld();
                float e8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) e8[i] = v[i] + v[8 + i];
                st_split8(sm + OFF_ET + ipl(j, 8 * sub, 0, C), C * 16, e8);
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                warp_arrive(bars.re, lane);
            }

            // ---- G: A_kk / A_qk(cn) from TMEM; the blocked triangular solve; T'
            if (prep) {
                if (!ptx::mbar_wait(bars.a, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
                ptx::tc_fence_after();
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + TM_A + 16 * sub, v);
                ptx::tmem_wait_ld();
                const float *sbeta = sbeta_all + (cn & 1) * C;
                if (lane < 16) {
                    const int row = 16 * quad + lane;   // M=64 rows sit in lanes 0-15 of each quadrant
                    if (row < C) {
                        const float br = sbeta[row];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int s = 8 * sub + i;
                            Akk[row * (C + 1) + s] = (s < row) ? br * (v[i] + v[8 + i]) : 0.f;
                        }
                    } else {
                        const int r = row - C;
                        float x[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) x[i] = (8 * sub + i <= r) ? v[i] + v[8 + i] : 0.f;
                        st_split8(sm + OFF_AQ + (cn & 1) * AQ_BYTES + ipl(r, 8 * sub, 0, C), C * 16, x);
                    }
                }
                ptx::tc_fence_before();
                cbar();
                blocked_solve(Akk, Ts, Tx, tid);
                if (tid < 128) {   // T' = T Diag(beta): row r, columns 8sc..8sc+7
                    const int r = tid >> 2, sc = tid & 3;
                    float x[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int s = 8 * sc + i;
                        x[i] = (sc > (r >> 3)) ? 0.f : Ts[r * (C + 1) + s] * sbeta[s];
                    }
                    st_split8(sm + OFF_TP + ipl(r, 8 * sc, 0, C), C * 16, x);
                }
                ptx::fence_proxy_async_smem();
                warp_arrive(bars.rg, lane);
            }

            // ---- I: state update of chunk c and its outputs; S'(cn) into TMEM
            if (chain) {
                if (!ptx::mbar_wait(bars.s, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
                ptx::tc_fence_after();
                const float *cst = reinterpret_cast<const float *>(sm + OFF_CST + (c & 1) * CST_BYTES);
                float v[32];
                ptx::tmem_ld32(tmem + lane_base + TM_S + 32 * sub, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = 32 * sub + i;
                    Sreg[i] = fmaf(cst[2 * D + d], Sreg[i], cst[D + d] * v[i]);
                }
                float o16[16];
                ptx::tmem_ld16(tmem + lane_base + TM_O + 16 * sub, o16);
                ptx::tmem_wait_ld();
                const int t0 = c * C;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * sub + i;
                    if (t0 + r < p.T) {
                        const size_t row = ((size_t)b * p.T + t0 + r) * p.H + h;
                        st_elem(p.o, row * D + j, o16[i] + o16[8 + i], p.out_bf16);
                    }
                }
            }
            if (prep) {
                // zero the O accumulator for the next chunk; S' = Diag(exp(a)) S as the
                // TMEM A operand (row j, K = d packed in pairs)
                ptx::tmem_st16_zero(tmem + lane_base + TM_O + 16 * sub);
                const float *cst = reinterpret_cast<const float *>(sm + OFF_CST + (cn & 1) * CST_BYTES);
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float x0 = cst[32 * sub + 2 * m] * Sreg[2 * m];
                    const float x1 = cst[32 * sub + 2 * m + 1] * Sreg[2 * m + 1];
                    __nv_bfloat16 h0, l0, h1, l1;
                    split2(x0, h0, l0);
                    split2(x1, h1, l1);
                    __nv_bfloat162 hp, lp;
                    hp.x = h0; hp.y = h1;
                    lp.x = l0; lp.y = l1;
                    hw[m] = *reinterpret_cast<uint32_t *>(&hp);
                    lw[m] = *reinterpret_cast<uint32_t *>(&lp);
                }
                ptx::tmem_st16(tmem + lane_base + TM_SP + 16 * sub, hw);
                ptx::tmem_st16(tmem + lane_base + TM_SP + 64 + 16 * sub, lw);
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();

            // ---- J: -W'(cn) from TMEM (lanes = key channel d) into rows 64..95 of the operand
            if (prep) {
                if (!ptx::mbar_wait(bars.w, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
                ptx::tc_fence_after();
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + TM_A + 16 * sub, v);
                ptx::tmem_wait_ld();
                const int d = j;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * sub + i;
                    __nv_bfloat16 hi, lo;
                    split2(-(v[i] + v[8 + i]), hi, lo);
                    const uint32_t off = ipl(2 * C + r, d, 0, D);
                    *reinterpret_cast<__nv_bfloat16 *>(lqr_n + off) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(lqr_n + off + D * 16) = lo;
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                warp_arrive(bars.rj, lane);
            }
            cbar();
            if (*err_flag) break;
        }

        if (p.s_out) {
            const size_t tile = (size_t)bh * D * D;
#pragma unroll
            for (int i = 0; i < 32; ++i) p.s_out[tile + (size_t)(32 * sub + i) * D + j] = Sreg[i];
        }
        ptx::cp_async_wait_all();
    }
    if (*err_flag && tid == 0 && p.status) atomicOr(p.status, 1u);
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
