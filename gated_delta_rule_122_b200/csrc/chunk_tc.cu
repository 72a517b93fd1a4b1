// Chunkwise KDA prefill on the sm_100a tensor cores (tcgen05, TMEM accumulators).
//
// Scope: d_k = d_v = 128, bf16 q/k/v, bf16 alpha/beta, fp32 state and output.
// One block per (sequence, head) walks chunks of C = 32 tokens with three warp
// roles: 8 "chain" warps run the serial inter-chunk recurrence and, between two
// state updates, build the decay-scaled operands of the chunk two ahead; 4 "prep"
// warps turn the A products into T' and W' for the next chunk at the same time;
// one warp's lane 0 issues every tcgen05.mma.
//
// Per chunk, with G[r] = sum_{t<=r} log alpha_t (per key channel), an anchor
// a = G[15] in the middle of the chunk and e_r = exp(G_r - a):
//   Lk = K*e, Lq = scale*Q*e, R = K/e            (bf16 hi/lo operands)
//   [A_kk; A_qk]  = [Lk; Lq] R^T                 (M=64 N=32 K=128)
//   A_kk <- strict lower * beta_r,  A_qk <- lower incl. diagonal
//   T'   = (I + A_kk)^-1 Diag(beta)              (blocked substitution, fp32)
//   W'^T = Lk^T T'^T,   U^T = V^T T'^T
// The state is carried pre-scaled, S' = Diag(exp(a)) S, which makes W S = W' S'
// and (scale Q gamma) S = Lq S' with gamma_r = exp(G_r) the pages' in-chunk
// decay.  Then
//   [O | E]^T = U^T + S'^T [Lq | -W']^T          (S' read from TMEM)
//   O^T += E^T A_qk^T
//   X^T  = S'^T + E^T R                          (accumulated onto S' in TMEM)
//   S_next = Diag(exp(G_end - a)) X,  S'_next = Diag(exp(a_next)) S_next
// since K*gamma_end/gamma = R Diag(exp(G_end - a)) and gamma_end = exp(a) *
// exp(G_end - a).  The anchor bounds every operand by exp(16 tokens of decay);
// products are the exact pairwise decays.
//
// Precision: operands that are not exact bf16 inputs are split x = hi + lo.
// Each product runs as two MMAs per K step, A_hi x [B_hi | B_lo] and
// A_lo x [B_hi | B_lo], the B planes concatenated along N, so the accumulator
// holds (hi + lo)(hi + lo) in two column groups summed when read.  Operands are
// "plane-interleaved": each 8-row block keeps its hi core matrices followed by
// its lo core matrices, so one buffer serves as a single-plane operand, as the
// two planes concatenated along N, and (swapping the descriptor strides) as
// the transposed operand.  The state update and all accumulations are fp32.
//
// The serial products are computed transposed: value channel j is the MMA's M
// index and TMEM lane; the fp32 state lives in TMEM.
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
constexpr int NCW = 8;           // chain warps (state recurrence, operand preparation)
constexpr int NCT = NCW * 32;
constexpr int NPW = 4;           // prep warps (A readout, solve, W' readout)
constexpr int NPT = NPW * 32;
constexpr int NT = NCT + NPT + 32;   // + the MMA-issuer warp
constexpr int kIssuerWarp = NCW + NPW;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait
constexpr int kChainBar = 1, kPrepBar = 2;         // named barriers of the two roles
constexpr int kCstSlots = 4;                       // per-chunk constants kept in flight

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
constexpr int OFF_CST = OFF_V + 2 * V_BYTES;           // kCstSlots x {exp(a), exp(G_end - a), f}[128]
constexpr int CST_BYTES = 3 * D * 4;                   // f(n) = exp(a_n) exp(G_end,n-1 - a_n-1)
constexpr int OFF_BETA = OFF_CST + kCstSlots * CST_BYTES;   // 2 x beta[32]
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
constexpr int NBARS = 9;
constexpr int OFF_BAR = OFF_TS + C * (C + 1) * 4;
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;          // tmem base, error flag
constexpr int SMEM_BYTES = OFF_MISC + 16;

// TMEM columns
constexpr uint32_t TM_A = 0;      // [A_kk; A_qk] (M=64 layout, N=64)
constexpr uint32_t TM_O = 64;     // O^T (64 cols: hi/lo groups), directly followed by
constexpr uint32_t TM_E = 128;    // E^T (64 cols) so that one N=128 MMA writes both
constexpr uint32_t TM_S = 192;    // fp32 S'^T, accumulated into X^T by the E^T R product
constexpr uint32_t TM_SP = 320;   // S'^T hi (64 cols) and lo (64 cols), the A operand of M3
constexpr uint32_t TM_W = 448;    // W'^T (N=64)
constexpr uint32_t TM_COLS = 512;

// x = hi + lo with hi = x truncated to bf16 (exact) and lo = bf16(x - hi); the
// pair carries ~16 significant bits.  Packs two values into a hi word and a lo word.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hw, uint32_t &lw)
{
    const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
    const float l0 = x0 - __uint_as_float(u0 & 0xFFFF0000u);
    const float l1 = x1 - __uint_as_float(u1 & 0xFFFF0000u);
    hw = __byte_perm(u0, u1, 0x7632);            // upper halves of u0 (low) and u1 (high)
    const __nv_bfloat162 lp = __floats2bfloat162_rn(l0, l1);
    lw = *reinterpret_cast<const uint32_t *>(&lp);
}

// Store 8 values (consecutive k) as hi and lo 16-byte chunks; lo sits plane_gap after hi.
__device__ __forceinline__ void st_split8(uint8_t *p, int plane_gap, const float (&x)[8])
{
    uint4 h, l;
    split_pair(x[0], x[1], h.x, l.x);
    split_pair(x[2], x[3], h.y, l.y);
    split_pair(x[4], x[5], h.z, l.z);
    split_pair(x[6], x[7], h.w, l.w);
    *reinterpret_cast<uint4 *>(p) = h;
    *reinterpret_cast<uint4 *>(p + plane_gap) = l;
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

__device__ __forceinline__ void chain_bar() { ptx::named_bar_sync(kChainBar, NCT); }
__device__ __forceinline__ void prep_bar() { ptx::named_bar_sync(kPrepBar, NPT); }

__device__ __forceinline__ float load_beta(const ChunkArgs &p, int b, int h, int n, int r)
{
    const int t = n * C + r;
    if (t >= p.T) return 0.f;
    return __bfloat162float(((const __nv_bfloat16 *)p.beta)[((size_t)b * p.T + t) * p.H + h]);
}

// Every warp of a role arrives once (barrier count = the role's warps).
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane)
{
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}

struct Bars {
    uint32_t a, w, e, s;      // issuer -> warps (tcgen05.commit)
    uint32_t rc, rs, re;      // chain -> issuer: operands staged, S' written, E^T written
    uint32_t rg, rj;          // prep -> issuer: T' and A_qk written, -W' written
};

// ---- the MMA-issuer warp (lane 0) -------------------------------------------------
// Four MMA groups per chunk: M1 (A-products) and M2 (W', U) depend only on the
// prep warps, M3 (O, E) and M4 (O, X) on the chain warps.  The issuer polls the
// readiness barriers and issues whichever group is ready next, so neither role
// waits behind the other's group.
__device__ void issuer(uint8_t *sm, uint32_t tmem, const Bars &bars, int nchunks, volatile int *err_flag)
{
    const uint32_t id_A = ptx::idesc_bf16(64, 64, 0, 0, 0);      // [Lk;Lq] x [R_hi|R_lo]
    const uint32_t id_W = ptx::idesc_bf16(128, 64, 1, 0, 0);     // Lk^T (MN view) x T'
    const uint32_t id_OE = ptx::idesc_bf16(128, 128, 0, 0, 0);   // S' x [Lq | -W']
    const uint32_t id_O2 = ptx::idesc_bf16(128, 64, 0, 0, 0);    // E^T x A_qk
    const uint32_t id_dS = ptx::idesc_bf16(128, 128, 0, 1, 0);   // E^T x R (MN view)
    int n1 = 0, n2 = 0, n3 = 0, n4 = 0;   // next chunk of each group
    uint64_t t_idle = ptx::global_timer_ns();
    while (n4 < nchunks) {
        bool issued = false;
        // M3(n3): needs S'(n3) (rs), W'(n3) (rj, also implies Lq(n3)), U(n3) (M2 issued)
        if (n3 < n2 && n3 <= n4 && ptx::mbar_test_wait(bars.rs, (uint32_t)(n3 & 1)) &&
            ptx::mbar_test_wait(bars.rj, (uint32_t)(n3 & 1))) {
            ptx::tc_fence_after();
            const uint32_t b0 = ptx::smem_u32(sm + OFF_LQR + (n3 & 1) * LQR_BYTES) + 4 * D * 32;
            for (int ks = 0; ks < D / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl)
                    ptx::mma_bf16_ts(tmem + TM_O, tmem + TM_SP + 64 * pl + 8 * ks,
                                     ptx::smem_desc(b0 + 256 * ks, 128, D * 16), id_OE, 1);
            ptx::mma_commit(bars.e);
            ++n3;
            issued = true;
        }
        // M4(n4): needs E^T(n4) (re)
        if (n4 < n3 && ptx::mbar_test_wait(bars.re, (uint32_t)(n4 & 1))) {
            ptx::tc_fence_after();
            const uint32_t et = ptx::smem_u32(sm + OFF_ET);
            const uint32_t aq = ptx::smem_u32(sm + OFF_AQ + (n4 & 1) * AQ_BYTES);
            const uint32_t rr = ptx::smem_u32(sm + OFF_LQR + (n4 & 1) * LQR_BYTES) + R_OFF;
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl)
                    ptx::mma_bf16(tmem + TM_O, ptx::smem_desc(et + C * 16 * pl + 256 * ks, 128, C * 32),
                                  ptx::smem_desc(aq + 256 * ks, 128, C * 16), id_O2, 1);
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pa = 0; pa < 2; ++pa)
                    for (int pb = 0; pb < 2; ++pb)
                        // R as the MN-major (N = d, K = s) operand: d-blocks 128 B apart,
                        // s-blocks (row-blocks) D*32 B apart
                        ptx::mma_bf16(tmem + TM_S,
                                      ptx::smem_desc(et + C * 16 * pa + 256 * ks, 128, C * 32),
                                      ptx::smem_desc(rr + D * 16 * pb + 2 * D * 32 * ks, D * 32, 128),
                                      id_dS, 1);
            ptx::mma_commit(bars.s);
            ++n4;
            issued = true;
        }
        // M1(n1): needs Lk, Lq, R of chunk n1 (rc; the prep warps read A(n1-1) before that)
        if (n1 < nchunks && n1 == n2 && ptx::mbar_test_wait(bars.rc, (uint32_t)(n1 & 1))) {
            ptx::tc_fence_after();
            const uint32_t lq = ptx::smem_u32(sm + OFF_LQR + (n1 & 1) * LQR_BYTES);
            const uint32_t rr = lq + R_OFF;
            uint32_t acc = 0;
            for (int ks = 0; ks < D / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl) {
                    ptx::mma_bf16(tmem + TM_A, ptx::smem_desc(lq + D * 16 * pl + 256 * ks, 128, D * 32),
                                  ptx::smem_desc(rr + 256 * ks, 128, D * 16), id_A, acc);
                    acc = 1;
                }
            ptx::mma_commit(bars.a);
            ++n1;
            issued = true;
        }
        // M2(n2): needs T', A_qk of chunk n2 (rg; the prep warps read W'(n2-1) before that);
        // writes U into TM_E, so E(n2-1) must be consumed (M4(n2-1) issued)
        if (n2 < n1 && n2 <= n4 && ptx::mbar_test_wait(bars.rg, (uint32_t)(n2 & 1))) {
            ptx::tc_fence_after();
            const uint32_t lk = ptx::smem_u32(sm + OFF_LQR + (n2 & 1) * LQR_BYTES);
            const uint32_t tp = ptx::smem_u32(sm + OFF_TP);
            const uint32_t vv = ptx::smem_u32(sm + OFF_V + (n2 & 1) * V_BYTES);
            uint32_t acc = 0;
            for (int ks = 0; ks < C / 16; ++ks)
                for (int pl = 0; pl < 2; ++pl) {
                    // Lk as the MN-major (M = d, K = s) operand
                    ptx::mma_bf16(tmem + TM_W,
                                  ptx::smem_desc(lk + D * 16 * pl + 2 * D * 32 * ks, D * 32, 128),
                                  ptx::smem_desc(tp + 256 * ks, 128, C * 16), id_W, acc);
                    acc = 1;
                }
            for (int ks = 0; ks < C / 16; ++ks)
                ptx::mma_bf16(tmem + TM_E, ptx::smem_desc(vv + 256 * ks, 128, (C / 8) * 128),
                              ptx::smem_desc(tp + 256 * ks, 128, C * 16), id_W, ks > 0);
            ptx::mma_commit(bars.w);
            ++n2;
            issued = true;
        }
        if (issued) {
            t_idle = ptx::global_timer_ns();
        } else {
            if (ptx::global_timer_ns() - t_idle > kWaitLimitNs || *err_flag) {
                *err_flag = 1;
                return;
            }
            __nanosleep(32);   // nothing ready: leave the issue slots to the compute warps
        }
    }
}

// ---- T' = (I + A_kk)^-1 Diag(beta) in one warp ---------------------------------------
// Lane c computes column c of T by right-looking forward substitution: once t_k
// is final, every later row's partial sum takes its A[i][k] t_k term, so the
// dependent chain is one FMA per row; A[i][k] are broadcast shared-memory reads.
// The column is transposed through shared memory and written as the K-major
// plane-interleaved B operand of M2 (rows r, K = s).
__device__ void solve_warp(const float *A, float *Ts, const float *sbeta, uint8_t *tp, int lane)
{
    constexpr int P = C + 1;
    float t[C];
#pragma unroll
    for (int i = 0; i < C; ++i) t[i] = (i == lane) ? 1.f : 0.f;
#pragma unroll
    for (int k = 0; k < C; ++k) {
        const float tk = t[k];
#pragma unroll
        for (int i = k + 1; i < C; ++i) t[i] = fmaf(-A[i * P + k], tk, t[i]);
    }
    const float bc = sbeta[lane];
#pragma unroll
    for (int r = 0; r < C; ++r) Ts[r * P + lane] = t[r] * bc;
    __syncwarp();
#pragma unroll
    for (int sc = 0; sc < 4; ++sc) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = Ts[lane * P + 8 * sc + i];
        st_split8(tp + ipl(lane, 8 * sc, 0, C), C * 16, x);
    }
}

// ---- operand preparation of chunk n (chain warps, between two state updates) -------
// Row r = lane, key channels 8g..8g+7 for g = warp, warp + 8: the prefix sum of
// log2 alpha over the chunk (a warp scan over rows), the anchored decays, the
// bf16 hi/lo operands Lk, Lq, R, and the chunk's per-channel constants.
__device__ void stage_operands(const ChunkArgs &p, uint8_t *sm, int n, int warp, int lane)
{
    const int r = lane;
    const int Lc = min(C, p.T - n * C);
    uint8_t *lqr = sm + OFF_LQR + (n & 1) * LQR_BYTES;
    float *cst = reinterpret_cast<float *>(sm + OFF_CST + (n % kCstSlots) * CST_BYTES);
    const float *cst_prev = reinterpret_cast<const float *>(sm + OFF_CST + ((n + kCstSlots - 1) % kCstSlots) * CST_BYTES);
#pragma unroll 1
    for (int gi = 0; gi < 2; ++gi) {
        const int g = warp + NCW * gi;        // key channels 8g .. 8g+7
        float q8[8], k8[8], x[8];
        ld_bf16x8(sm + OFF_STG + STG_Q + r * ROWB + g * 16, q8);
        ld_bf16x8(sm + OFF_STG + STG_K + r * ROWB + g * 16, k8);
        ld_bf16x8(sm + OFF_STG + STG_A + r * ROWB + g * 16, x);
        // base-2 log of the retention, floored at 2^-115.4 (= e^-80); rows past the
        // end are identity steps
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = (r < Lc) ? fmaxf(ptx::lg2(x[i]), -115.4f) : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float y = __shfl_up_sync(0xffffffffu, x[i], off);
                if (lane >= off) x[i] += y;
            }
        }
        float lk[8], lq[8], rk[8], my_a = 0.f, my_gl = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a = __shfl_sync(0xffffffffu, x[i], 15);
            const float gl = __shfl_sync(0xffffffffu, x[i], 31);
            if (lane == i) { my_a = a; my_gl = gl; }
            const float t = fminf(fmaxf(x[i] - a, -125.f), 125.f);
            const float e = ptx::ex2(t), re = ptx::ex2(-t);
            lk[i] = k8[i] * e;
            lq[i] = p.scale * q8[i] * e;
            rk[i] = k8[i] * re;
        }
        if (lane < 8) {
            const int d = 8 * g + lane;
            const float aexp = ptx::ex2(fmaxf(my_a, -125.f));
            cst[d] = aexp;                                                     // exp(a)
            cst[D + d] = ptx::ex2(fminf(fmaxf(my_gl - my_a, -125.f), 125.f));  // exp(G_end - a)
            cst[2 * D + d] = (n > 0) ? aexp * cst_prev[D + d] : 0.f;           // state-update factor
        }
        st_split8(lqr + ipl(r, 8 * g, 0, D), D * 16, lk);
        st_split8(lqr + ipl(C + r, 8 * g, 0, D), D * 16, lq);
        st_split8(lqr + R_OFF + ipl(r, 8 * g, 0, D), D * 16, rk);
    }
}

// cp.async copies of chunk n's q, k, alpha rows into the staging rows (chain warps).
__device__ void prefetch_qka(const ChunkArgs &p, uint8_t *sm, int b, int h, int n, int ct)
{
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t HD = (size_t)p.H * D;
#pragma unroll
    for (int it = 0; it < 6; ++it) {
        const int idx = ct + it * NCT;          // 0..1535; tensor = it / 2
        const int rem = idx & 511;
        const int r = rem >> 4, ch = rem & 15;
        const int rr = r < L ? r : 0;
        const uint32_t nbytes = r < L ? 16u : 0u;
        const size_t g = ((size_t)b * p.T + t0 + rr) * HD + (size_t)h * D + ch * 8;
        const int tensor = it >> 1;
        const void *src = tensor == 0 ? (const void *)((const __nv_bfloat16 *)p.q + g)
                        : tensor == 1 ? (const void *)((const __nv_bfloat16 *)p.k + g)
                                      : (const void *)((const __nv_bfloat16 *)p.alpha + g);
        ptx::cp_async16(ptx::smem_u32(sm + OFF_STG + tensor * C * ROWB + r * ROWB + ch * 16), src, nbytes);
    }
    ptx::cp_async_commit();
}

// cp.async copies of chunk n's v rows into V buffer n&1, MN-major (prep warps).
__device__ void prefetch_v(const ChunkArgs &p, uint8_t *sm, int b, int h, int n, int pt)
{
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t HD = (size_t)p.H * D;
    uint8_t *vb = sm + OFF_V + (n & 1) * V_BYTES;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int rem = pt + it * NPT;          // 0..511
        const int r = rem >> 4, ch = rem & 15;
        const int rr = r < L ? r : 0;
        const size_t g = ((size_t)b * p.T + t0 + rr) * HD + (size_t)h * D + ch * 8;
        ptx::cp_async16(ptx::smem_u32(vb + mnmaj(ch * 8, r, C)), (const __nv_bfloat16 *)p.v + g,
                        r < L ? 16u : 0u);
    }
    ptx::cp_async_commit();
}

// ---- the prep warps: A readout, the solve, W' readout, V loads ---------------------
__device__ void prep_role(const ChunkArgs &p, uint8_t *sm, uint32_t tmem, const Bars &bars, int b, int h,
                          int nchunks, volatile int *err_flag)
{
    const int pt = threadIdx.x - NCT;          // 0..127
    const int pw = pt >> 5, lane = pt & 31;    // warp = TMEM lane quadrant
    const uint32_t lane_base = (uint32_t)(pw * 32) << 16;
    float *Akk = reinterpret_cast<float *>(sm + OFF_AKK);
    float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
    float *sbeta_all = reinterpret_cast<float *>(sm + OFF_BETA);

    prefetch_v(p, sm, b, h, 0, pt);
    if (nchunks > 1) prefetch_v(p, sm, b, h, 1, pt);
    if (pw == 0) sbeta_all[lane] = load_beta(p, b, h, 0, lane);
    prep_bar();

    for (int cn = 0; cn < nchunks; ++cn) {
        const float *sbeta = sbeta_all + (cn & 1) * C;
        // beta of the next chunk, stored once this chunk's A readout is done (warp 0
        // ran the solve of chunk cn-1 that read the same slot)
        const float beta_next = (pw == 0 && cn + 1 < nchunks) ? load_beta(p, b, h, cn + 1, lane) : 0.f;

        // ---- G(cn): A_kk / A_qk from TMEM; the solve in warp 0; T'
        if (!ptx::mbar_wait(bars.a, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
#pragma unroll 1
        for (int hs = 0; hs < 2; ++hs) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + TM_A + 32 * hs, v);
            ptx::tmem_wait_ld();
            if (lane < 16) {
                const int row = 16 * pw + lane;   // M=64 rows sit in lanes 0-15 of each quadrant
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int sb = 2 * hs + u;       // s = 8sb .. 8sb+7
                    if (row < C) {
                        const float br = sbeta[row];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int s = 8 * sb + i;
                            Akk[row * (C + 1) + s] = (s < row) ? br * (v[16 * u + i] + v[16 * u + 8 + i]) : 0.f;
                        }
                    } else {
                        const int r = row - C;
                        float x[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            x[i] = (8 * sb + i <= r) ? v[16 * u + i] + v[16 * u + 8 + i] : 0.f;
                        st_split8(sm + OFF_AQ + (cn & 1) * AQ_BYTES + ipl(r, 8 * sb, 0, C), C * 16, x);
                    }
                }
            }
        }
        if (pw == 0) sbeta_all[((cn + 1) & 1) * C + lane] = beta_next;
        ptx::cp_async_wait_all();            // V(cn) (and V(cn+1)) have landed
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        prep_bar();
        if (pw == 0) {
            solve_warp(Akk, Ts, sbeta, sm + OFF_TP, lane);
            ptx::fence_proxy_async_smem();
            warp_arrive(bars.rg, lane);
        }

        // ---- J(cn): -W' from TMEM (lanes = key channel d) into rows 64..95 of the operand
        if (!ptx::mbar_wait(bars.w, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            uint8_t *lqr = sm + OFF_LQR + (cn & 1) * LQR_BYTES;
            const int d = 32 * pw + lane;
#pragma unroll 1
            for (int hs = 0; hs < 2; ++hs) {
                float v[32];
                ptx::tmem_ld32(tmem + lane_base + TM_W + 32 * hs, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        uint32_t hw, lw;
                        split_pair(-(v[16 * u + i] + v[16 * u + 8 + i]), -(v[16 * u + i + 1] + v[16 * u + 9 + i]), hw, lw);
                        const int r = 16 * hs + 8 * u + i;
                        const uint32_t off0 = ipl(2 * C + r, d, 0, D), off1 = ipl(2 * C + r + 1, d, 0, D);
                        *reinterpret_cast<uint16_t *>(lqr + off0) = (uint16_t)(hw & 0xFFFFu);
                        *reinterpret_cast<uint16_t *>(lqr + off1) = (uint16_t)(hw >> 16);
                        *reinterpret_cast<uint16_t *>(lqr + off0 + D * 16) = (uint16_t)(lw & 0xFFFFu);
                        *reinterpret_cast<uint16_t *>(lqr + off1 + D * 16) = (uint16_t)(lw >> 16);
                    }
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        warp_arrive(bars.rj, lane);
        // M2(cn) has completed: its V buffer can take chunk cn+2
        if (cn + 2 < nchunks) prefetch_v(p, sm, b, h, cn + 2, pt);
        if (*err_flag) break;
    }
    ptx::cp_async_wait_all();
}

// 16 columns of S'^T in this thread's row j, starting at key channel d0: scale
// the fp32 values, write them back, and write the bf16 hi/lo planes of the M3
// operand (two bf16 per TMEM column).
__device__ __forceinline__ void write_state16(uint32_t tmem, uint32_t lane_base, int d0, float (&v)[16],
                                              const float *scale_d)
{
    uint32_t fw[16], hw[8], lw[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[i] *= scale_d[i];
        fw[i] = __float_as_uint(v[i]);
    }
    ptx::tmem_st16(tmem + lane_base + TM_S + d0, fw);
#pragma unroll
    for (int m = 0; m < 8; ++m) split_pair(v[2 * m], v[2 * m + 1], hw[m], lw[m]);
    ptx::tmem_st8(tmem + lane_base + TM_SP + d0 / 2, hw);
    ptx::tmem_st8(tmem + lane_base + TM_SP + 64 + d0 / 2, lw);
}

// Chain warps: stage chunk n's operands (staging must hold chunk n) and signal the
// issuer; then start loading chunk n+1 into the staging rows.
__device__ void chain_prepare(const ChunkArgs &p, uint8_t *sm, const Bars &bars, int b, int h, int n,
                              int nchunks, int tid, int warp, int lane)
{
    ptx::cp_async_wait_all();
    chain_bar();
    stage_operands(p, sm, n, warp, lane);
    ptx::fence_proxy_async_smem();
    warp_arrive(bars.rc, lane);
    chain_bar();   // staging consumed, constants visible to every chain warp
    if (n + 1 < nchunks) prefetch_qka(p, sm, b, h, n + 1, tid);
}

// ---- the chain warps: the serial recurrence over chunks --------------------------------
__device__ void chain_role(const ChunkArgs &p, uint8_t *sm, uint32_t tmem, const Bars &bars, int b, int h,
                           int bh, int nchunks, volatile int *err_flag)
{
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int j = quad * 32 + lane;            // value channel = TMEM lane
    const size_t tile = (size_t)bh * D * D;

    prefetch_qka(p, sm, b, h, 0, tid);
    chain_prepare(p, sm, bars, b, h, 0, nchunks, tid, warp, lane);

    // S'_0 = Diag(exp(a_0)) S_0; cleared O accumulator
    {
        const float *cst0 = reinterpret_cast<const float *>(sm + OFF_CST);
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
            const int d0 = 64 * half + 16 * part;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = p.s_in ? p.s_in[tile + (size_t)(d0 + i) * D + j] : 0.f;
            write_state16(tmem, lane_base, d0, v, cst0 + d0);
        }
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half);
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half + 16);
        ptx::tmem_wait_st();
    }
    ptx::tc_fence_before();
    warp_arrive(bars.rs, lane);
    if (nchunks > 1) chain_prepare(p, sm, bars, b, h, 1, nchunks, tid, warp, lane);

    for (int c = 0; c < nchunks; ++c) {
        // ---- E: E^T = U^T - S'^T W'^T (hi and lo groups) into the A operand of M4
        if (!ptx::mbar_wait(bars.e, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + TM_E + 32 * half, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float e8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) e8[i] = v[16 * u + i] + v[16 * u + 8 + i];
                st_split8(sm + OFF_ET + ipl(j, 8 * (2 * half + u), 0, C), C * 16, e8);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        warp_arrive(bars.re, lane);

        // ---- I: X = S' + E^T R -> the next S' (or the final state); outputs of chunk c
        if (!ptx::mbar_wait(bars.s, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        float ov[16];
        {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + TM_O + 32 * half, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) ov[8 * u + i] = v[16 * u + i] + v[16 * u + 8 + i];
        }
        if (c + 1 < nchunks) {
            // f(c+1) = exp(a_{c+1}) exp(G_end,c - a_c), written when chunk c+1 was staged
            const float *f = reinterpret_cast<const float *>(sm + OFF_CST + ((c + 1) % kCstSlots) * CST_BYTES) + 2 * D;
            ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half);
            ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half + 16);
#pragma unroll 1
            for (int part = 0; part < 4; ++part) {
                const int d0 = 64 * half + 16 * part;
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + TM_S + d0, v);
                ptx::tmem_wait_ld();
                write_state16(tmem, lane_base, d0, v, f + d0);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            warp_arrive(bars.rs, lane);
        } else if (p.s_out) {
            const float *cend = reinterpret_cast<const float *>(sm + OFF_CST + (c % kCstSlots) * CST_BYTES) + D;
#pragma unroll 1
            for (int part = 0; part < 4; ++part) {
                const int d0 = 64 * half + 16 * part;
                float v[16];
                ptx::tmem_ld16(tmem + lane_base + TM_S + d0, v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) p.s_out[tile + (size_t)(d0 + i) * D + j] = cend[d0 + i] * v[i];
            }
        }
        {
            const int t0 = c * C;
            const size_t step = (size_t)p.H * D;
            size_t idx = (((size_t)b * p.T + t0 + 16 * half) * p.H + h) * D + j;
#pragma unroll
            for (int i = 0; i < 16; ++i, idx += step)
                if (t0 + 16 * half + i < p.T) st_elem(p.o, idx, ov[i], p.out_bf16);
        }
        // ---- operands of chunk c+2 (its operand stage held chunk c, whose MMAs are done)
        if (c + 2 < nchunks) chain_prepare(p, sm, bars, b, h, c + 2, nchunks, tid, warp, lane);
        if (*err_flag) break;
    }
    ptx::cp_async_wait_all();
}

__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(ChunkArgs p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int nchunks = (p.T + C - 1) / C;

    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *err_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const uint32_t bar0 = ptx::smem_u32(sm + OFF_BAR);
    Bars bars;
    bars.a = bar0; bars.w = bar0 + 8; bars.e = bar0 + 16; bars.s = bar0 + 24;
    bars.rc = bar0 + 32; bars.rg = bar0 + 40; bars.rj = bar0 + 48;
    bars.rs = bar0 + 56; bars.re = bar0 + 64;

    if (tid == 0) {
        ptx::mbar_init(bars.a, 1);
        ptx::mbar_init(bars.w, 1);
        ptx::mbar_init(bars.e, 1);
        ptx::mbar_init(bars.s, 1);
        ptx::mbar_init(bars.rc, NCW);
        ptx::mbar_init(bars.rg, 1);
        ptx::mbar_init(bars.rj, NPW);
        ptx::mbar_init(bars.rs, NCW);
        ptx::mbar_init(bars.re, NCW);
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

    if (warp == kIssuerWarp) {
        if (lane == 0) issuer(sm, tmem, bars, nchunks, err_flag);
    } else if (warp >= NCW) {
        prep_role(p, sm, tmem, bars, b, h, nchunks, err_flag);
    } else {
        chain_role(p, sm, tmem, bars, b, h, bh, nchunks, err_flag);
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
