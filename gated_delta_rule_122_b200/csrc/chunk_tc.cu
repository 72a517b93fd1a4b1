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
//   [A_kk; A_qk]  = [Lk; Lq] R^T                 (one M=128 product over both planes)
//   A_kk <- strict lower * beta_r,  A_qk <- lower incl. diagonal
//   T'   = (I + A_kk)^-1 Diag(beta)              (substitution in one warp, fp32)
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
// products are the exact pairwise decays.  e and 1/e are running products of
// alpha away from the anchor row (no logarithms), floored at 2^-125.
//
// Precision: operands that are not exact bf16 inputs are split x = hi + lo and
// every product sums all four hi/lo cross terms: the planes are either
// concatenated along M or N of one MMA (summed when the accumulator is read)
// or issued as two MMAs into the same accumulator.  The state update and all
// accumulations are fp32.
//
// Layouts.  Lk, Lq, R and -W' are stored "d-major": 2 KB slabs of 8 rows
// (tokens) x 128 key channels, each 16-byte core-matrix row holding 8
// consecutive tokens of one channel.  The same slab is a K-major operand when
// channels index M/N (W', X products) and an MN-major operand when tokens do
// (A products, the O/E product), and one thread per channel writes it with
// 16-byte stores.  The serial products are computed transposed: value channel j
// is the MMA's M index and TMEM lane; the fp32 state lives in TMEM.
//
// Algorithm: "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two schedules for
// the same recurrence"; "From Fast Weight Programmers to KDA"
// (jonahsamost.bearblog.dev), section "Kimi Delta Attention".
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cstring>
#include <mutex>

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
// The chain thread that issues the staging loads, their L2 prefetches and the output
// stores: lane 0 of the last chain warp, whose SM sub-partition does not also run the
// MMA-issuer warp (warps are spread over the four sub-partitions by index mod 4).
constexpr int kTmaThread = NCT - 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait
constexpr int kChainBar = 1, kPrepBar = 2;         // named barriers of the two roles
constexpr int kCstSlots = 4;                       // per-chunk constants kept in flight
constexpr float kMinAlpha = 1.8048513e-35f;        // e^-80: per-token retention floor
constexpr float kMinScale = 2.3509887e-38f;        // 2^-125: floor of the anchored decays
// A chunk in which some key channel decays by more than 2^-100 over one 16-token half
// (about 69 nats) is outside the range in which the anchored factors e and 1/e, and
// their products with the operands, are exact in fp32.  Such a chunk is computed token
// by token instead (the sequential form of the recurrence, fp32, on the chain warps).
constexpr float kExtremeDecay = 7.8886091e-31f;    // 2^-100
constexpr float kExtremeInv = 1.2676506e30f;       // 2^100

// ---- operand layouts ----------------------------------------------------------------
// d-major slab (8 tokens x 128 channels, 2 KB): channel block d/8 at 128 B, channel
// d%8 at 16 B, token r%8 at 2 B.
constexpr int SLAB = 2048;
__device__ __forceinline__ uint32_t dm(int slab, int d, int r)
{
    return (uint32_t)(slab * SLAB + (d >> 3) * 128 + (d & 7) * 16 + (r & 7) * 2);
}
// Slabs of one operand stage: every operand keeps token block rb's hi plane in slab
// base + 2rb and its lo plane in base + 2rb + 1.  M=128 A-product operand = slabs
// 0..15 (Lk, Lq), O/E product operand = slabs 8..23 (Lq, -W'), R = slabs 24..31.
constexpr int SL_LK = 0, SL_LQ = 8, SL_W = 16, SL_R = 24;

// Plane-interleaved K-major layout with K = 32 (E^T: rows j; T', A_qk: rows r;
// K = s): row block row/8 holds the hi plane's 4 core matrices, then the lo
// plane's, so the N = 64 operand [rows 0-7 hi, rows 0-7 lo, rows 8-15 hi, ...]
// has uniform 512-byte row-block strides.
__device__ __forceinline__ uint32_t ipl(int row, int k, int plane)
{
    return (uint32_t)((row >> 3) * (C * 32) + plane * (C * 16) + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}
// Plain MN-major layout (V): core matrices (mn/8, k/8) at (mn/8)*(K/8)*128 + (k/8)*128.
__device__ __forceinline__ uint32_t mnmaj(int mn, int k, int K)
{
    return (uint32_t)((mn >> 3) * (K / 8) * 128 + (k >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2);
}

// ---- shared-memory plan (bytes) ----------------------------------------------------
// q, k, alpha of one chunk are staged as dense 256-byte rows (one TMA box each).
__device__ __forceinline__ int stg_row(int r) { return r * 256; }
constexpr int STG_T = C * 256;                         // one staged tensor
constexpr int OFF_STG = 0;                             // staged q, k, alpha of one chunk
constexpr int STG_Q = 0, STG_K = STG_T, STG_A = 2 * STG_T;
constexpr int OFF_V = OFF_STG + 3 * STG_T;             // 2 x V (A of U^T: M=j, K=s, MN-major)
constexpr int V_BYTES = D * C * 2;
constexpr int OFF_CST = OFF_V + 2 * V_BYTES;           // kCstSlots x {exp(a), exp(G_end - a), f}[128]
constexpr int CST_BYTES = 3 * D * 4;                   // f(n) = exp(a_n) exp(G_end,n-1 - a_n-1)
constexpr int OFF_LQR = (OFF_CST + kCstSlots * CST_BYTES + 127) / 128 * 128;   // 2 operand stages
constexpr int LQR_BYTES = 32 * SLAB;
constexpr int OFF_ET = OFF_LQR + 2 * LQR_BYTES;        // E^T (A of the O and X products)
constexpr int OFF_TP = OFF_ET + D * C * 4;             // T'  (B of W'/U: N = r, K = s)
constexpr int OFF_AQ = OFF_TP + C * C * 4;             // 2 x A_qk (B of O: N = r, K = s)
constexpr int AQ_BYTES = C * C * 4;
constexpr int P = C + 1;                               // fp32 [32][33] tiles
constexpr int OFF_XS = OFF_AQ + 2 * AQ_BYTES;          // A10 T0 of the solve fp32 [16][33]
constexpr int OFF_AKK = OFF_XS + C * P * 4;            // A_kk^T fp32 [32][36]
constexpr int OFF_TS = OFF_AKK + C * (C + 4) * 4;      // T fp32 [32][33]
constexpr int OFF_BETA = OFF_TS + C * P * 4;           // beta of the chunk being solved
// raw inputs: 1/||q_r||, 1/||k_r|| of a chunk, a ring of kNrmSlots chunks (stage A writes
// chunk n, the prep warps and the chain's E and O readouts of chunk n read it)
constexpr int kNrmSlots = 4;
constexpr int NRM_BYTES = 2 * C * 4;
constexpr int OFF_NRM = OFF_BETA + C * 4;
constexpr int OFF_TPU = (OFF_NRM + kNrmSlots * NRM_BYTES + 127) / 128 * 128;   // raw: T Diag(beta), B of U
constexpr int NBARS = 14;
constexpr int OFF_BAR = (OFF_TPU + C * C * 4 + 7) / 8 * 8;
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;          // tmem base, error flag
// Chunks whose decay leaves the range of the anchored factors: slot n % 4 holds n + 1
// when chunk n is one (written by stage A, read by the chain warps after a barrier).
constexpr int kXSlots = 4;
constexpr int OFF_XF = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_XF + 4 * kXSlots;
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds the per-block limit");
static_assert(OFF_AKK % 16 == 0 && OFF_LQR % 128 == 0 && OFF_TP % 128 == 0 && OFF_TPU % 128 == 0,
              "vector and operand alignment");

// TMEM columns
constexpr uint32_t TM_A = 0;      // [A_kk; A_qk] per plane of Lk, Lq (M=128, N=64)
constexpr uint32_t TM_O = 64;     // O^T (64 cols: hi/lo groups), directly followed by
constexpr uint32_t TM_E = 128;    // E^T (64 cols) so that one N=128 MMA writes both
constexpr uint32_t TM_S = 192;    // fp32 S'^T, accumulated into X^T by the E^T R product
constexpr uint32_t TM_SP = 320;   // S'^T hi (64 cols) and lo (64 cols), the A operand of M3
constexpr uint32_t TM_W = 448;    // W'^T (N=64: T' hi rows, then lo rows)
constexpr uint32_t TM_COLS = 512;

// x = hi + lo with hi = x truncated to bf16 (exact) and lo = bf16(x - hi); the
// pair carries ~16 significant bits.  Packs two values into a hi word and a lo word.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hw, uint32_t &lw)
{
    const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
    float l0, l1;
    ptx::upk2(ptx::sub2(ptx::pk2(x0, x1), ptx::pk2(__uint_as_float(u0 & 0xFFFF0000u), __uint_as_float(u1 & 0xFFFF0000u))),
              l0, l1);
    hw = __byte_perm(u0, u1, 0x7632);            // upper halves of u0 (low) and u1 (high)
    const __nv_bfloat162 lp = __floats2bfloat162_rn(l0, l1);
    lw = *reinterpret_cast<const uint32_t *>(&lp);
}

// Store 8 values as hi and lo 16-byte chunks; lo sits plane_gap bytes after hi.
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

__device__ __forceinline__ float ld_bf16(const uint8_t *p)
{
    return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t *>(p)) << 16);
}

__device__ __forceinline__ void chain_bar() { ptx::named_bar_sync(kChainBar, NCT); }
__device__ __forceinline__ void prep_bar() { ptx::named_bar_sync(kPrepBar, NPT); }
// The same barriers, returning whether any thread of the role has seen the error
// flag: a role leaves its loop only on this common answer, so no thread is left
// waiting at a named barrier (which has no time limit).
__device__ __forceinline__ bool chain_bar_err(volatile int *err_flag)
{
    return ptx::named_bar_sync_or(kChainBar, NCT, *err_flag != 0);
}
__device__ __forceinline__ bool prep_bar_err(volatile int *err_flag)
{
    return ptx::named_bar_sync_or(kPrepBar, NPT, *err_flag != 0);
}

template <bool kRaw, bool kGdn2 = false>
__device__ __forceinline__ float load_beta(const ChunkArgs &p, const SeqSpan &sp, int h, int n, int r)
{
    const int t = n * C + r;
    if (t >= sp.len) return 0.f;
    if constexpr (kGdn2) return 1.f;   // GDN-2: the write gate takes beta's place, on v
    const float y = __bfloat162float(((const __nv_bfloat16 *)p.beta)[(sp.tok0 + t) * p.H + h]);
    if constexpr (kRaw) return ptx::rcp(1.f + __expf(-y));   // a beta logit: sigmoid(y)
    else return y;
}

// TMA descriptors of one launch: q, k, alpha as [B][T][H][128] boxes of 32 token
// rows; v as the 5-D view (j%8, t, j/8, h, b) whose 8 x 32 x 16 box lands in the
// MN-major core-matrix layout of the U^T product; o as boxes of 16 token rows.
struct TcMaps {
    CUtensorMap q, k, a, v, o;
    CUtensorMap w, b;   // GDN-2: write gate (as v) and erase gate (as k, L2 prefetches only)
};
constexpr int HG_ROW = 16;   // bytes per token row of a staged per-head gate box

// The gate kind is a template parameter of the kernel (a run-time choice inside stage A
// costs the chain measurably): alpha rows per token and key channel, one gate per
// (token, head) staged by TMA as boxes of 8 heads x 32 tokens, or read from memory.
// kGateGdn2: alpha per key channel plus GDN-2's erase gate b [B, T, H, d_k] (the
// retrieval key is b * k) and write gate w [B, T, H, d_v] (the target is w * v), no beta
// ("From Fast Weight Programmers to KDA", section "Gated DeltaNet-2").
constexpr int kGateChannel = 0, kGateHeadTma = 1, kGateHeadMem = 2, kGateGdn2 = 3;
__host__ __device__ constexpr bool per_channel(int g) { return g == kGateChannel || g == kGateGdn2; }

// Every warp of a role arrives once on a readiness mbarrier once its writes are visible
// (release semantics; the barrier's phase for chunk n completes when all the role's
// warps have arrived, and the MMA issuer waits on it with acquire semantics).
__device__ __forceinline__ void warp_signal(uint32_t bar, int lane)
{
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}

struct Bars {
    uint32_t a, w, e, s;      // issuer -> warps (mbarriers, tcgen05.commit)
    uint32_t stg, v;          // TMA fills: q/k/alpha staging; V buffers (v and v + 8)
    // warps -> issuer (mbarriers, one arrival per warp and chunk):
    uint32_t rc;              // chain: operands of chunk n staged (rc + 8 (n & 1): one per parity of n)
    uint32_t rs, re;          // chain: S' written, E^T written
    uint32_t ra, rg, rj;      // prep: A read, T' and A_qk written, -W' written
};

// ---- the MMA-issuer warp (lane 0) -------------------------------------------------
// Four MMA groups per chunk: M1 (A-products) and M2 (W', U) depend only on the
// prep warps, M3 (O, E) and M4 (O, X) on the chain warps.  The tensor pipe runs
// them in issue order.  The issuer polls the readiness counters (plain shared
// loads) and issues the most urgent ready group: the chain's M3 and M4 first,
// then M2, then M1.
struct MmaIds {
    uint32_t A, W, U, OE, O2, dS;
};

// Descriptor of the operand bytes further on than desc's: the start address field holds
// address / 16 in its low 14 bits, and every operand here lies below 256 KB of shared
// memory, so the step is a plain add (built once per group, not once per MMA).
__device__ __forceinline__ uint64_t desc_at(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

__device__ __forceinline__ void issue_m3(uint8_t *sm, uint32_t tmem, const Bars &bars, const MmaIds &id, int n3)
{
    ptx::tc_fence_after();
    const uint64_t lq = ptx::smem_desc(ptx::smem_u32(sm + OFF_LQR + (n3 & 1) * LQR_BYTES) + SL_LQ * SLAB, 128, SLAB);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
            ptx::mma_bf16_ts(tmem + TM_O, tmem + TM_SP + 64 * pl + 8 * ks, desc_at(lq, 256 * ks), id.OE, 1);
    ptx::mma_commit(bars.e);
}

__device__ __forceinline__ void issue_m4(uint8_t *sm, uint32_t tmem, const Bars &bars, const MmaIds &id, int n4)
{
    ptx::tc_fence_after();
    const uint64_t et = ptx::smem_desc(ptx::smem_u32(sm + OFF_ET), 128, C * 32);
    const uint64_t aq = ptx::smem_desc(ptx::smem_u32(sm + OFF_AQ + (n4 & 1) * AQ_BYTES), 128, 512);
    const uint64_t rr =
        ptx::smem_desc(ptx::smem_u32(sm + OFF_LQR + (n4 & 1) * LQR_BYTES) + SL_R * SLAB, 2 * SLAB, 128);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks)
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
            ptx::mma_bf16(tmem + TM_O, desc_at(et, C * 16 * pl + 256 * ks), desc_at(aq, 256 * ks), id.O2, 1);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks)
#pragma unroll
        for (int pa = 0; pa < 2; ++pa)
#pragma unroll
            for (int pb = 0; pb < 2 - pa; ++pb)
                // R as the K-major (N = d, K = s) operand: token blocks 2 slabs apart.  The
                // E_lo R_lo term (2^-16 of the product) is left out: three cross terms.
                ptx::mma_bf16(tmem + TM_S, desc_at(et, C * 16 * pa + 256 * ks),
                              desc_at(rr, SLAB * pb + 4 * SLAB * ks), id.dS, 1);
    ptx::mma_commit(bars.s);
}

__device__ __forceinline__ void issue_m1(uint8_t *sm, uint32_t tmem, const Bars &bars, const MmaIds &id, int n1)
{
    ptx::tc_fence_after();
    const uint32_t base = ptx::smem_u32(sm + OFF_LQR + (n1 & 1) * LQR_BYTES);
    const uint64_t lk = ptx::smem_desc(base + SL_LK * SLAB, 128, SLAB), r = ptx::smem_desc(base + SL_R * SLAB, 128, SLAB);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
        ptx::mma_bf16(tmem + TM_A, desc_at(lk, 256 * ks), desc_at(r, 256 * ks), id.A, ks > 0);
    ptx::mma_commit(bars.a);
}

template <int kGate, bool kRaw>
__device__ __forceinline__ void issue_m2(uint8_t *sm, uint32_t tmem, const Bars &bars, const MmaIds &id, int n2)
{
    ptx::tc_fence_after();
    const uint64_t lk = ptx::smem_desc(ptx::smem_u32(sm + OFF_LQR + (n2 & 1) * LQR_BYTES) + SL_LK * SLAB, 2 * SLAB, 128);
    const uint64_t tp = ptx::smem_desc(ptx::smem_u32(sm + OFF_TP), 128, 512);
    // GDN-2: one V stage holding the hi and lo planes of w * v in the two V buffers
    const uint64_t vv = ptx::smem_desc(ptx::smem_u32(sm + OFF_V + (kGate == kGateGdn2 ? 0 : (n2 & 1) * V_BYTES)), 128,
                                       (C / 8) * 128);
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks)
#pragma unroll
        for (int pl = 0; pl < 2; ++pl)
            // Lk plane pl as the K-major (M = d, K = s) operand: token blocks 2 slabs apart
            ptx::mma_bf16(tmem + TM_W, desc_at(lk, pl * SLAB + 4 * SLAB * ks), desc_at(tp, 256 * ks), id.W,
                          ks > 0 || pl > 0);
    // raw inputs: T Diag(beta) for U
    const uint64_t tu = kRaw ? ptx::smem_desc(ptx::smem_u32(sm + OFF_TPU), 128, 512) : tp;
    constexpr int kVPlanes = kGate == kGateGdn2 ? 2 : 1;
#pragma unroll
    for (int ks = 0; ks < C / 16; ++ks)
#pragma unroll
        for (int pl = 0; pl < kVPlanes; ++pl)
            ptx::mma_bf16(tmem + TM_E, desc_at(vv, pl * V_BYTES + 256 * ks), desc_at(tu, 256 * ks), id.U,
                          ks > 0 || pl > 0);
    ptx::mma_commit(bars.w);
}

// The issuer takes the groups in a fixed order, waiting on each group's readiness
// mbarriers (the warp sleeps in the wait and wakes when the phase completes):
//   M1(0), M1(1), M2(0), then for each chunk c: M3(c), M4(c), M2(c+1), M1(c+2)
// (with R staged after the state rewrite: M1(0), M2(0), then M3(c), M1(c+1), M4(c), M2(c+1)).
// M1(n) needs Lk, Lq, R of chunk n (rc) and A(n-1) read by the prep warps (ra, since
// A(n) overwrites it); M2(n) needs T' and A_qk (rg, which the prep warps signal after
// reading W'(n-1)) and the E readout of chunk n-1 (U(n) overwrites E in TMEM; implied
// by M4(n-1) having been issued); M3(n) needs S'(n) (rs) and -W'(n) (rj); M4(n) needs
// E^T(n) (re).  Each producer is at most one phase ahead of this order: every arrival
// for chunk n+1 depends on a group of chunk n that is issued after the wait for chunk n.
template <int kGate, bool kRaw, bool kLateB>
__device__ void issuer(uint8_t *sm, uint32_t tmem, const Bars &bars, int nchunks, volatile int *err_flag)
{
    MmaIds id;
    id.A = ptx::idesc_bf16(128, 64, 1, 1, 0);     // [Lk; Lq] (MN) x R (MN)
    id.W = ptx::idesc_bf16(128, 64, 0, 0, 0);     // Lk (d x s) x T'
    id.U = ptx::idesc_bf16(128, 64, 1, 0, 0);     // V (MN) x T'
    id.OE = ptx::idesc_bf16(128, 128, 0, 1, 0);   // S' (TMEM) x [Lq | -W'] (MN)
    id.O2 = ptx::idesc_bf16(128, 64, 0, 0, 0);    // E^T x A_qk
    id.dS = ptx::idesc_bf16(128, 128, 0, 0, 0);   // E^T x R (d x s)
    bool ok = true;
    auto wait = [&](uint32_t bar, int phase) {
        if (ok && !ptx::mbar_wait(bar, (uint32_t)(phase & 1), kWaitLimitNs)) ok = false;
        return ok;
    };
    // M1(n): operands of chunk n staged (rc, one barrier per parity of n) and A(n-1) read
    auto m1 = [&](int n) {
        if (n > 0) wait(bars.ra, n - 1);
        if (wait(bars.rc + 8 * (n & 1), n >> 1)) issue_m1(sm, tmem, bars, id, n);
    };
    auto m2 = [&](int n) {
        if (wait(bars.rg, n)) issue_m2<kGate, kRaw>(sm, tmem, bars, id, n);
    };
    // kLateB (R staged after the state rewrite, so that rc(c+2) arrives after rs(c+1)):
    // M3(c), M1(c+1), M4(c), M2(c+1), so that M3(c+1) does not queue behind M1(c+2)
    m1(0);
    if (!kLateB && nchunks > 1) m1(1);
    m2(0);
    for (int c = 0; c < nchunks && ok; ++c) {
        wait(bars.rs, c);
        if (wait(bars.rj, c)) issue_m3(sm, tmem, bars, id, c);
        if (kLateB && c + 1 < nchunks) m1(c + 1);
        if (wait(bars.re, c)) issue_m4(sm, tmem, bars, id, c);
        if (c + 1 < nchunks) m2(c + 1);
        if (!kLateB && c + 2 < nchunks) m1(c + 2);
        if (*err_flag) ok = false;
    }
    if (!ok) *err_flag = 1;
}

// ---- T' = (I + A_kk)^-1 Diag(beta), blocked over the four prep warps -------------
// With A = [[A00, 0], [A10, A11]] in 16x16 blocks, (I + A)^-1 = [[T0, 0],
// [-T1 A10 T0, T1]] with T0 = (I + A00)^-1 and T1 = (I + A11)^-1.  One warp
// computes T0 (lanes 0-15) and T1 (lanes 16-31) at once, lane = column, by
// right-looking forward substitution; A is stored transposed (At[k][i]) so a
// column is read as broadcast 16-byte loads.  All four warps then form
// X = A10 T0 and T10 = -T1 X, two entries per thread, and write T' = T Diag(beta)
// as the plane-major K-major B operand of M2 (rows r, K = s).
constexpr int PT = C + 4;   // row pitch of At (16-byte aligned rows)
__device__ __forceinline__ void solve_diag_blocks(const float *At, float *Tm, int lane)
{
    const int c = lane & 15, off = lane & 16;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = (i == c) ? 1.f : 0.f;
#pragma unroll
    for (int k = 0; k < 15; ++k) {
        const float tk = t[k];
#pragma unroll
        for (int i4 = (k + 1) / 4; i4 < 4; ++i4) {
            const float4 a = *reinterpret_cast<const float4 *>(At + (off + k) * PT + off + 4 * i4);
            if (4 * i4 + 0 > k) t[4 * i4 + 0] = fmaf(-a.x, tk, t[4 * i4 + 0]);
            if (4 * i4 + 1 > k) t[4 * i4 + 1] = fmaf(-a.y, tk, t[4 * i4 + 1]);
            if (4 * i4 + 2 > k) t[4 * i4 + 2] = fmaf(-a.z, tk, t[4 * i4 + 2]);
            if (4 * i4 + 3 > k) t[4 * i4 + 3] = fmaf(-a.w, tk, t[4 * i4 + 3]);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tm[(off + i) * P + off + c] = t[i];
}

// ---- operand preparation of chunk n (chain warps) -----------------------------------
// Thread (warp w, lane): key channel d = 32(w%4) + lane, token rows 16h..16h+15
// with h = w/4.  Away from the anchor row 15 the decays are running products of
// alpha: for r >= 16, e_r = prod_{16..r} alpha; for r < 16, 1/e_r =
// prod_{r+1..15} alpha, so each half of the chunk is self-contained.  Part A
// writes Lk, Lq and the chunk constants and returns 1/e; part B writes R = K/e.
// Part A only touches slabs the A product (M1), the W'/U product (M2) and the O/E
// product (M3) of the chunk two back have finished with, so it can run while that
// chunk's state update (M4) still reads R.
template <int kGate, bool kRaw>
__device__ void stage_a(const ChunkArgs &p, uint8_t *sm, const SeqSpan &sp, int h, int n, int warp, int lane,
                        uint32_t (&rw)[16])
{
    const int hf = warp >> 2, d = 32 * (warp & 3) + lane;
    const int Lc = min(C, sp.len - n * C);
    uint8_t *lqr = sm + OFF_LQR + (n & 1) * LQR_BYTES;
    float *cst = reinterpret_cast<float *>(sm + OFF_CST + (n % kCstSlots) * CST_BYTES);
    const float *cst_prev = reinterpret_cast<const float *>(sm + OFF_CST + ((n + kCstSlots - 1) % kCstSlots) * CST_BYTES);
    const uint8_t *stg = sm + OFF_STG;
    // alpha of row r: the staged row's channel d, or with one gate per head, the token's
    // gate straight from global memory (the same 32 values for every thread)
    const __nv_bfloat16 *ah = (const __nv_bfloat16 *)p.alpha + (sp.tok0 + (size_t)n * C) * p.H + h;
    auto alpha_at = [&](int r) {
        if constexpr (kGate == kGateHeadTma) return ld_bf16(stg + STG_A + HG_ROW * r + 2 * (h & 7));
        else if constexpr (kGate == kGateHeadMem) return __bfloat162float(ah[(size_t)r * p.H]);
        else return ld_bf16(stg + STG_A + stg_row(r) + 2 * d);
    };
    // Per-token factor of the running products: alpha (floored at e^-80), or with a gate
    // logit x its inverse 1/alpha = 1 + e^x (capped at e^80): the products then hold the
    // inverse decays, and the one reciprocal per row below gives the other side, so the
    // logit costs one exponential and no reciprocal.
    auto factor = [&](int r) {
        if constexpr (kRaw) return fminf(1.f + __expf(alpha_at(r)), 1.f / kMinAlpha);
        else return fmaxf(alpha_at(r), kMinAlpha);
    };
    float pr[16];
    float acc = 1.f;
    if (hf == 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 + i;
            acc *= (r < Lc) ? factor(r) : 1.f;             // rows past the end: identity steps
            pr[i] = acc;                                     // e_r (raw: 1/e_r)
        }
        cst[D + d] = fmaxf(kRaw ? ptx::rcp(acc) : acc, kMinScale);   // exp(G_end - a)
        if (kRaw ? !(acc <= kExtremeInv) : !(acc >= kExtremeDecay))
            reinterpret_cast<volatile int *>(sm + OFF_XF)[n % kXSlots] = n + 1;
    } else {
#pragma unroll
        for (int i = 15; i >= 0; --i) {
            pr[i] = acc;                                     // 1/e_r (raw: e_r)
            acc *= (i < Lc) ? factor(i) : 1.f;
        }
        const float aexp = fmaxf(kRaw ? ptx::rcp(acc) : acc, kMinScale);   // exp(a)
        if (kRaw ? !(acc <= kExtremeInv) : !(acc >= kExtremeDecay))
            reinterpret_cast<volatile int *>(sm + OFF_XF)[n % kXSlots] = n + 1;
        cst[d] = aexp;
        cst[2 * D + d] = (n > 0) ? aexp * cst_prev[D + d] : 0.f;   // state-update factor
    }
    const bool e_in_pr = (hf == 1) != kRaw;   // pr holds e (else 1/e)
    // GDN-2: the erase gate of this channel for the chunk's rows, read from global memory
    // (prefetched to L2 with the staged rows)
    const __nv_bfloat16 *bcol =
        kGate == kGateGdn2 ? (const __nv_bfloat16 *)p.erase + ((sp.tok0 + (size_t)n * C) * p.H + h) * D + d : nullptr;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        float lk[8], lq[8], ie[8], bv[8];
        if constexpr (kGate == kGateGdn2) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 16 * hf + 8 * u + i;
                bv[i] = (r < Lc) ? __bfloat162float(bcol[(size_t)r * p.H * D]) : 0.f;
            }
        }
        const uint64_t scale2 = ptx::pk2(p.scale, p.scale);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            float e[2], kv[2], qv[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int r = 16 * hf + 8 * u + i + t;
                const float m = fminf(fmaxf(pr[8 * u + i + t], kMinScale), 1.f / kMinScale);
                const float rm = ptx::rcp(m);
                e[t] = e_in_pr ? m : rm;
                ie[i + t] = e_in_pr ? rm : m;
                // rows past the sequence's end: zero (the staging may hold another sequence's rows)
                kv[t] = (r < Lc) ? ld_bf16(stg + STG_K + stg_row(r) + 2 * d) : 0.f;
                qv[t] = (r < Lc) ? ld_bf16(stg + STG_Q + stg_row(r) + 2 * d) : 0.f;
            }
            const uint64_t e2 = ptx::pk2(e[0], e[1]);
            if constexpr (kGate == kGateGdn2)   // the retrieval key b * k
                ptx::upk2(ptx::mul2(ptx::mul2(ptx::pk2(kv[0], kv[1]), ptx::pk2(bv[i], bv[i + 1])), e2), lk[i], lk[i + 1]);
            else
                ptx::upk2(ptx::mul2(ptx::pk2(kv[0], kv[1]), e2), lk[i], lk[i + 1]);
            ptx::upk2(ptx::mul2(ptx::mul2(ptx::pk2(qv[0], qv[1]), scale2), e2), lq[i], lq[i + 1]);
            // R = K/e, kept split (hi words, lo words) until its slabs are free
            float r0, r1;
            ptx::upk2(ptx::mul2(ptx::pk2(kv[0], kv[1]), ptx::pk2(ie[i], ie[i + 1])), r0, r1);
            split_pair(r0, r1, rw[8 * u + i / 2], rw[8 * u + 4 + i / 2]);
        }
        st_split8(lqr + dm(SL_LK + 2 * (2 * hf + u), d, 0), SLAB, lk);
        st_split8(lqr + dm(SL_LQ + 2 * (2 * hf + u), d, 0), SLAB, lq);
    }
}

__device__ void stage_b(uint8_t *sm, int n, int warp, int lane, const uint32_t (&rw)[16])
{
    const int hf = warp >> 2, d = 32 * (warp & 3) + lane;
    uint8_t *lqr = sm + OFF_LQR + (n & 1) * LQR_BYTES;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        uint8_t *dst = lqr + dm(SL_R + 2 * (2 * hf + u), d, 0);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(rw[8 * u], rw[8 * u + 1], rw[8 * u + 2], rw[8 * u + 3]);
        *reinterpret_cast<uint4 *>(dst + SLAB) = make_uint4(rw[8 * u + 4], rw[8 * u + 5], rw[8 * u + 6], rw[8 * u + 7]);
    }
}

// Where a sequence's rows sit in the tensor maps: batch coordinate b and first token
// t0 (b = sequence, t0 = 0 for the dense layout; b = 0, t0 = its offset when packed).
struct TmaPos {
    int b, h, t0;
};

// TMA loads of chunk n's q, k, alpha rows into the staging rows (one thread).  Rows
// past the sequence's end are masked where they are used.
template <int kGate>
__device__ __forceinline__ void load_qka(const TcMaps &maps, uint8_t *sm, const Bars &bars, const TmaPos &tp, int n)
{
    const uint32_t dst = ptx::smem_u32(sm + OFF_STG);
    ptx::mbar_arrive_expect_tx(bars.stg, 2 * STG_T + (per_channel(kGate) ? STG_T : kGate == kGateHeadTma ? C * HG_ROW : 0));
    ptx::tma_load_4d(dst + STG_Q, &maps.q, bars.stg, 0, tp.h, tp.t0 + n * C, tp.b);
    ptx::tma_load_4d(dst + STG_K, &maps.k, bars.stg, 0, tp.h, tp.t0 + n * C, tp.b);
    if constexpr (per_channel(kGate)) ptx::tma_load_4d(dst + STG_A, &maps.a, bars.stg, 0, tp.h, tp.t0 + n * C, tp.b);
    // heads h & ~7 .. (h & ~7) + 7 of 32 tokens: the x coordinate is a multiple of 8 elements
    if constexpr (kGate == kGateHeadTma) ptx::tma_load_3d(dst + STG_A, &maps.a, bars.stg, tp.h & ~7, tp.t0 + n * C, tp.b);
}

// L2 prefetch of chunk n's q, k, alpha rows (one thread), issued a few chunks before the
// staging load of the same rows so that the load finds them in L2.
template <int kGate>
__device__ __forceinline__ void prefetch_qka(const TcMaps &maps, const TmaPos &tp, int n)
{
    ptx::tma_prefetch_4d(&maps.q, 0, tp.h, tp.t0 + n * C, tp.b);
    ptx::tma_prefetch_4d(&maps.k, 0, tp.h, tp.t0 + n * C, tp.b);
    if constexpr (per_channel(kGate)) ptx::tma_prefetch_4d(&maps.a, 0, tp.h, tp.t0 + n * C, tp.b);
    if constexpr (kGate == kGateGdn2) ptx::tma_prefetch_4d(&maps.b, 0, tp.h, tp.t0 + n * C, tp.b);
    if constexpr (kGate == kGateHeadTma) ptx::tma_prefetch_3d(&maps.a, tp.h & ~7, tp.t0 + n * C, tp.b);
}

// TMA load of chunk n's v rows into V buffer n&1 (one thread).  GDN-2: v into the first
// buffer and the write gate w into the second (one stage, refilled once M2 has read it;
// the prep warps turn the pair into the hi and lo planes of w * v in place).
template <int kGate>
__device__ __forceinline__ void load_v(const TcMaps &maps, uint8_t *sm, const Bars &bars, const TmaPos &tp, int n)
{
    if constexpr (kGate == kGateGdn2) {
        ptx::mbar_arrive_expect_tx(bars.v, 2 * V_BYTES);
        ptx::tma_load_5d(ptx::smem_u32(sm + OFF_V), &maps.v, bars.v, 0, tp.t0 + n * C, 0, tp.h, tp.b);
        ptx::tma_load_5d(ptx::smem_u32(sm + OFF_V + V_BYTES), &maps.w, bars.v, 0, tp.t0 + n * C, 0, tp.h, tp.b);
    } else {
        const uint32_t bar = bars.v + 8 * (n & 1);
        ptx::mbar_arrive_expect_tx(bar, V_BYTES);
        ptx::tma_load_5d(ptx::smem_u32(sm + OFF_V + (n & 1) * V_BYTES), &maps.v, bar, 0, tp.t0 + n * C, 0, tp.h, tp.b);
    }
}
// The mbarrier and phase parity of chunk n's V load.
template <int kGate>
__device__ __forceinline__ void v_bar(const Bars &bars, int n, uint32_t &bar, uint32_t &parity)
{
    if constexpr (kGate == kGateGdn2) {
        bar = bars.v;
        parity = (uint32_t)(n & 1);
    } else {
        bar = bars.v + 8 * (n & 1);
        parity = (uint32_t)((n >> 1) & 1);
    }
}

// ---- the prep warps: A readout, the solve, W' readout, V loads ---------------------
// The A product's four row groups (TMEM lane quadrants) are Lk_lo, Lk_hi, Lq_hi and
// Lq_lo times R: warps 0 and 2 hand their partial sums to warps 1 and 3 through
// shared memory; warp 1 forms A_kk and solves its diagonal blocks, warp 3 writes
// A_qk, and all four finish the off-diagonal block of T and write T'.
template <int kGate, bool kRaw>
__device__ void prep_role(const ChunkArgs &p, const TcMaps &maps, uint8_t *sm, uint32_t tmem, const Bars &bars,
                          const TmaPos &tp, const SeqSpan &sp, int h, int nchunks, volatile int *err_flag)
{
    const int pt = threadIdx.x - NCT;          // 0..127
    const int pw = pt >> 5, lane = pt & 31;    // warp = TMEM lane quadrant
    const uint32_t lane_base = (uint32_t)(pw * 32) << 16;
    float *At = reinterpret_cast<float *>(sm + OFF_AKK);   // A_kk transposed
    float *Tm = reinterpret_cast<float *>(sm + OFF_TS);    // T = (I + A_kk)^-1
    float *Xs = reinterpret_cast<float *>(sm + OFF_XS);    // A10 T0
    float *sbeta = reinterpret_cast<float *>(sm + OFF_BETA);
    // This lane's row of the A product: lane quadrant pw holds token blocks 2(pw&1)
    // and 2(pw&1)+1 of Lk (pw < 2) or Lq (pw >= 2), hi plane in lanes 0-7 / 16-23,
    // lo plane in lanes 8-15 / 24-31.
    const int pl = (lane >> 3) & 1;
    const int r = 16 * (pw & 1) + 8 * (lane >> 4) + (lane & 7);

    constexpr bool kGdn2 = kGate == kGateGdn2;
    constexpr int kVAhead = kGdn2 ? 1 : 2;   // V stages: GDN-2 uses both buffers for one chunk
    int v_loaded = 0, v_seen = 0;   // V loads issued (thread pt 0) and waited for
    if (pt == 0) {
        load_v<kGate>(maps, sm, bars, tp, 0);
        if (!kGdn2 && nchunks > 1) load_v<kGate>(maps, sm, bars, tp, 1);
    }
    v_loaded = min(kVAhead, nchunks);
    float beta = (pw < 2) ? load_beta<kRaw, kGdn2>(p, sp, h, 0, r) : 0.f;   // beta of row r

    for (int cn = 0; cn < nchunks; ++cn) {
        const float beta_next = (pw < 2 && cn + 1 < nchunks) ? load_beta<kRaw, kGdn2>(p, sp, h, cn + 1, r) : 0.f;

        // ---- G(cn): A_kk / A_qk from TMEM; the solve; T'
        if (!ptx::mbar_wait(bars.a, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        // raw inputs: the chain's stage A of chunk cn wrote its norms before adding to the
        // count rc, which M1(cn) waited for; acquiring rc makes them visible here
        if constexpr (kRaw)
            if (!ptx::mbar_wait(bars.rc + 8 * (cn & 1), (uint32_t)((cn >> 1) & 1), kWaitLimitNs)) *err_flag = 1;
        float a32[32];   // this plane's row r times R, summed over R's planes
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
            float v[32];
            ptx::tmem_ld32(tmem + lane_base + TM_A + 32 * hs, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) a32[16 * hs + 8 * u + i] = v[16 * u + i] + v[16 * u + 8 + i];
        }
        ptx::tc_fence_before();
        warp_signal(bars.ra, lane);
        // add the other plane's row (lane ^ 8): this lane keeps columns s = 16 pl .. 16 pl + 15
        float ar[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float send = pl ? a32[i] : a32[16 + i];
            const float keep = pl ? a32[16 + i] : a32[i];
            ar[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        // V(cn) has landed (every warp observes it before it signals M2's readiness)
        {
            uint32_t vbar, vpar;
            v_bar<kGate>(bars, cn, vbar, vpar);
            if (!ptx::mbar_wait(vbar, vpar, kWaitLimitNs)) *err_flag = 1;
        }
        v_seen = cn + 1;
        uint8_t *vb = sm + OFF_V + (kGdn2 ? 0 : (cn & 1) * V_BYTES);
        if (sp.len - cn * C < C) {
            // rows past the sequence's end hold zeros (dense layout) or the next
            // sequence's tokens (packed): clear them, T' does not see them anyway
            const int Lc = sp.len - cn * C;
            for (int i = pt; i < (C - Lc) * (D / 8); i += NPT) {
                const int r = Lc + i / (D / 8), jb = i % (D / 8);
                *reinterpret_cast<uint4 *>(vb + mnmaj(8 * jb, r, C)) = make_uint4(0u, 0u, 0u, 0u);
            }
            if (kGdn2) prep_bar();   // the cleared rows before the products below read them
            ptx::fence_proxy_async_smem();
        }
        if constexpr (kGdn2) {
            // w * v in place: the first buffer holds v, the second w (the same MN-major
            // layout); they become the hi plane (w v truncated to bf16) and the lo plane
            // (bf16 of the rest), the two A operands of U
            for (int i = pt; i < V_BYTES / 16; i += NPT) {
                uint4 &hv = reinterpret_cast<uint4 *>(vb)[i];
                uint4 &lw = reinterpret_cast<uint4 *>(vb + V_BYTES)[i];
                const uint4 vv = hv, ww = lw;
                const uint32_t va[4] = {vv.x, vv.y, vv.z, vv.w}, wa[4] = {ww.x, ww.y, ww.z, ww.w};
                uint32_t ho[4], lo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = __uint_as_float(va[q] << 16) * __uint_as_float(wa[q] << 16);
                    const float x1 = __uint_as_float(va[q] & 0xFFFF0000u) * __uint_as_float(wa[q] & 0xFFFF0000u);
                    split_pair(x0, x1, ho[q], lo[q]);
                }
                hv = make_uint4(ho[0], ho[1], ho[2], ho[3]);
                lw = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            ptx::fence_proxy_async_smem();
        }
        if (pw < 2) {
            // A_kk^T: row r of A_kk scaled by beta_r, strictly lower (raw inputs: and by
            // nk_r nk_s)
            float rs = beta;
            const float *nk = reinterpret_cast<const float *>(sm + OFF_NRM + (cn % kNrmSlots) * NRM_BYTES) + C;
            if constexpr (kRaw) rs *= nk[r];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s = 16 * pl + i;
                const float cs = kRaw ? nk[s] : 1.f;
                At[s * PT + r] = (s < r) ? rs * cs * ar[i] : 0.f;
            }
            if (pl == 0) sbeta[r] = beta;
        } else {
            // A_qk row r, lower triangle including the diagonal
            uint8_t *aq = sm + OFF_AQ + (cn & 1) * AQ_BYTES;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = (16 * pl + 8 * u + i <= r) ? ar[8 * u + i] : 0.f;
                st_split8(aq + ipl(r, 16 * pl + 8 * u, 0), C * 16, x);
            }
            ptx::fence_proxy_async_smem();
        }
        prep_bar();
        if (pw == 1) solve_diag_blocks(At, Tm, lane);
        prep_bar();
        {
            // X = A10 T0 (rows 16..31 of A, columns 0..15), two columns per thread
            const int i = pt >> 3, c0 = 2 * (pt & 7);
            float x0 = 0.f, x1 = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float a = At[k * PT + 16 + i];
                x0 = fmaf(a, Tm[k * P + c0], x0);
                x1 = fmaf(a, Tm[k * P + c0 + 1], x1);
            }
            Xs[i * P + c0] = x0;
            Xs[i * P + c0 + 1] = x1;
            prep_bar();
            // T10 = -T1 X (T1 is lower triangular, stored with zeros above its diagonal)
            float y0 = 0.f, y1 = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float t1 = Tm[(16 + i) * P + 16 + k];
                y0 = fmaf(t1, Xs[k * P + c0], y0);
                y1 = fmaf(t1, Xs[k * P + c0 + 1], y1);
            }
            Tm[(16 + i) * P + c0] = -y0;
            Tm[(16 + i) * P + c0 + 1] = -y1;
        }
        const bool stop = prep_bar_err(err_flag);
        {
            // T' = T Diag(beta): row rt, columns 8sc..8sc+7, as hi/lo planes (raw inputs:
            // T Diag(beta nk) for W', and T Diag(beta) for U in its own buffer)
            const int rt = 8 * pw + (lane & 7), sc = lane >> 3;
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int s = 8 * sc + i;
                x[i] = (rt < 16 && s >= 16) ? 0.f : Tm[rt * P + s] * sbeta[s];
            }
            if constexpr (kRaw) {
                st_split8(sm + OFF_TPU + ipl(rt, 8 * sc, 0), C * 16, x);
                const float *nk = reinterpret_cast<const float *>(sm + OFF_NRM + (cn % kNrmSlots) * NRM_BYTES) + C;
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] *= nk[8 * sc + i];
            }
            st_split8(sm + OFF_TP + ipl(rt, 8 * sc, 0), C * 16, x);
            ptx::fence_proxy_async_smem();
        }
        warp_signal(bars.rg, lane);
        beta = beta_next;

        // ---- J(cn): -W' from TMEM (lanes = key channel d) into the W' slabs
        if (!ptx::mbar_wait(bars.w, (uint32_t)(cn & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        {
            uint8_t *lqr = sm + OFF_LQR + (cn & 1) * LQR_BYTES;
            const int d = 32 * pw + lane;
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                float v0[16], v1[16];   // token blocks 2hs and 2hs+1: T' hi rows, then lo rows
                ptx::tmem_ld16(tmem + lane_base + TM_W + 32 * hs, v0);
                ptx::tmem_ld16(tmem + lane_base + TM_W + 32 * hs + 16, v1);
                ptx::tmem_wait_ld();
                float x0[8], x1[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    x0[i] = -(v0[i] + v0[8 + i]);
                    x1[i] = -(v1[i] + v1[8 + i]);
                }
                st_split8(lqr + dm(SL_W + 2 * (2 * hs), d, 0), SLAB, x0);
                st_split8(lqr + dm(SL_W + 2 * (2 * hs + 1), d, 0), SLAB, x1);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        warp_signal(bars.rj, lane);
        // M2(cn) has completed: its V buffer can take chunk cn+2 (GDN-2: the one stage, cn+1)
        if (cn + kVAhead < nchunks) {
            if (pt == 0) load_v<kGate>(maps, sm, bars, tp, cn + kVAhead);
            v_loaded = cn + kVAhead + 1;
        }
        if (stop) break;
    }
    // on an early exit, let the V loads still in flight land before the block ends
    for (int n = v_seen; n < v_loaded; ++n) {
        uint32_t vbar, vpar;
        v_bar<kGate>(bars, n, vbar, vpar);
        (void)ptx::mbar_wait(vbar, vpar, kWaitLimitNs);
    }
}

// 16 columns of S'^T in this thread's row j, starting at key channel d0: scale
// the fp32 values, write them back, and write the bf16 hi/lo planes of the M3
// operand (two bf16 per TMEM column).
__device__ __forceinline__ void write_state16(uint32_t tmem, uint32_t lane_base, int d0, float (&v)[16],
                                              const float *scale_d, bool unscaled = false)
{
    uint32_t fw[16], hw[8], lw[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (!unscaled) v[i] *= scale_d[i];
        fw[i] = __float_as_uint(v[i]);
    }
    ptx::tmem_st16(tmem + lane_base + TM_S + d0, fw);
#pragma unroll
    for (int m = 0; m < 8; ++m) split_pair(v[2 * m], v[2 * m + 1], hw[m], lw[m]);
    ptx::tmem_st8(tmem + lane_base + TM_SP + d0 / 2, hw);
    ptx::tmem_st8(tmem + lane_base + TM_SP + 64 + d0 / 2, lw);
}

// Chain warps, operands of chunk n (the staging rows must hold chunk n): part A,
// then (later) part B, the signal to the issuer and the loads of chunk n+1.
// Raw inputs: 1/||q_r|| and 1/||k_r|| of chunk n's staged rows (0 past the sequence's
// end) into the norm ring, four rows of each per chain warp.  Each lane sums the squares
// of four channels; a transposed butterfly then reduces the eight rows together (over
// lane bits 4, 3, 2 each lane keeps half of its sums and adds its partner's matching
// half, ending with sum (lane >> 2) & 7; bits 1, 0 finish it), nine shuffles in all.  The factors
// are applied after the products, where each one is a row or column scaling:
//   A_kk -> Diag(nk) A_kk Diag(nk) and W' -> T Diag(beta nk) Lk (prep warps),
//   the E operand of the state update and of O -> Diag(nk) E, O -> Diag(nq) O (chain),
// so stage A itself is unchanged and needs no barrier.
__device__ __forceinline__ void row_norms(uint8_t *sm, int n, int len, int warp, int lane)
{
    const uint8_t *stg = sm + OFF_STG;
    auto sq4 = [&](int off, int r) {   // this lane's four channels of a staged row, squared and summed
        const uint2 w = *reinterpret_cast<const uint2 *>(stg + off + stg_row(r) + 8 * lane);
        const float a0 = __uint_as_float(w.x << 16), a1 = __uint_as_float(w.x & 0xFFFF0000u);
        const float a2 = __uint_as_float(w.y << 16), a3 = __uint_as_float(w.y & 0xFFFF0000u);
        return fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, a3 * a3)));
    };
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float w4[4], w2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float vq = sq4(STG_Q, 4 * warp + i), vk = sq4(STG_K, 4 * warp + i);
        w4[i] = (b4 ? vk : vq) + __shfl_xor_sync(0xffffffffu, b4 ? vq : vk, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
        w2[i] = (b3 ? w4[2 + i] : w4[i]) + __shfl_xor_sync(0xffffffffu, b3 ? w4[i] : w4[2 + i], 8);
    float w1 = (b2 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? w2[0] : w2[1], 4);
    w1 += __shfl_xor_sync(0xffffffffu, w1, 2);
    w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
    if ((lane & 3) == 0) {
        const int idx = lane >> 2, r = 4 * warp + (idx & 3);
        reinterpret_cast<float *>(sm + OFF_NRM + (n % kNrmSlots) * NRM_BYTES)[(idx < 4 ? 0 : C) + r] =
            (n * C + r < len) ? inv_norm(w1) : 0.f;
    }
}

template <int kGate, bool kRaw>
__device__ __forceinline__ void chain_stage_a(const ChunkArgs &p, uint8_t *sm, const Bars &bars, const SeqSpan &sp, int h, int n, int warp,
                                              int lane, uint32_t (&ie)[16], volatile int *err_flag)
{
    if (!ptx::mbar_wait(bars.stg, (uint32_t)(n & 1), kWaitLimitNs)) *err_flag = 1;   // chunk n's rows
    if constexpr (kRaw) row_norms(sm, n, sp.len, warp, lane);
    stage_a<kGate, kRaw>(p, sm, sp, h, n, warp, lane, ie);
}

template <int kGate>
__device__ __forceinline__ void chain_stage_b(const TcMaps &maps, uint8_t *sm, const Bars &bars, const TmaPos &tp,
                                              int n, int nchunks, int tid, int warp, int lane,
                                              const uint32_t (&ie)[16])
{
    stage_b(sm, n, warp, lane, ie);
    ptx::fence_proxy_async_smem();
    warp_signal(bars.rc + 8 * (n & 1), lane);
    chain_bar();   // staging consumed, constants visible to every chain warp
    if (tid == kTmaThread && n + 1 < nchunks) load_qka<kGate>(maps, sm, bars, tp, n + 1);
}

__device__ __forceinline__ void warp_signal_after_stage(const Bars &bars, int n, int lane)
{
    ptx::fence_proxy_async_smem();
    warp_signal(bars.rc + 8 * (n & 1), lane);
}

__device__ __forceinline__ bool chunk_is_extreme(const uint8_t *sm, int n)
{
    return reinterpret_cast<const volatile int *>(sm + OFF_XF)[n % kXSlots] == n + 1;
}

// Eight consecutive bf16 values (16 bytes) widened to fp32.
__device__ __forceinline__ void ld_bf16x8(const void *p, float (&x)[8])
{
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(u[i] << 16);
        x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// A chunk whose decay leaves the range of the anchored factors, token by token on the
// chain warps: the five-step update of each token in fp32.  This thread's part of the
// state, S[64 half + i][j] for i < 64 (key channels 64 half .. 64 half + 63 of value
// channel j), stays in its TMEM lane at columns TM_S + 64 half + i and is walked in two
// groups of 32 per pass.  The two predictions S~^T k, S~^T q and k.q are summed over the
// two halves through shared memory, one barrier per token; o_t = scale (S~^T q + e (k.q))
// is the read of S_t = S~ + k e^T.  Retention factors are used as they are (alpha = 0
// clears a channel exactly).  xb: 2 x 2 x 4 x 128 floats of scratch.
template <int kGate, bool kRaw>
__device__ __forceinline__ void sequential_chunk(const ChunkArgs &p, const uint8_t *sm, uint32_t tcol,
                                                 const SeqSpan &sp, int h, int c, int half, int j, float *xb)
{
    const int d0 = 64 * half;
    const int Lc = min(C, sp.len - c * C);
    const float *nrm = reinterpret_cast<const float *>(sm + OFF_NRM + (c % kNrmSlots) * NRM_BYTES);
#pragma unroll 1
    for (int r = 0; r < Lc; ++r) {
        const size_t row = (sp.tok0 + (size_t)c * C + r) * p.H + h;
        const __nv_bfloat16 *qr = (const __nv_bfloat16 *)p.q + row * D + d0;
        const __nv_bfloat16 *kr = (const __nv_bfloat16 *)p.k + row * D + d0;
        const __nv_bfloat16 *ar = (const __nv_bfloat16 *)p.alpha + row * D + d0;
        const __nv_bfloat16 *br = (const __nv_bfloat16 *)p.erase + row * D + d0;   // GDN-2 erase gate
        float ah = 1.f;   // one gate per (token, head)
        if constexpr (!per_channel(kGate)) ah = __bfloat162float(((const __nv_bfloat16 *)p.alpha)[row]);
        float pv = 0.f, pq = 0.f, kq = 0.f;
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            float sv[32];
            ptx::tmem_ld32(tcol + 32 * q2, sv);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float qv[8], kv[8], av[8], bv[8];
                ld_bf16x8(qr + 32 * q2 + 8 * g, qv);
                ld_bf16x8(kr + 32 * q2 + 8 * g, kv);
                if constexpr (per_channel(kGate)) ld_bf16x8(ar + 32 * q2 + 8 * g, av);
                if constexpr (kGate == kGateGdn2) ld_bf16x8(br + 32 * q2 + 8 * g, bv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float al = per_channel(kGate) ? av[i] : ah;
                    if constexpr (kRaw) al = 1.f / (1.f + __expf(al));   // gate logit x: alpha = 1/(1 + e^x)
                    float &x = sv[8 * g + i];
                    x *= al;
                    // the retrieval key: b * k for GDN-2
                    pv = fmaf(kGate == kGateGdn2 ? bv[i] * kv[i] : kv[i], x, pv);
                    pq = fmaf(qv[i], x, pq);
                    kq = fmaf(kv[i], qv[i], kq);
                }
            }
            ptx::tmem_st32(tcol + 32 * q2, sv);
        }
        ptx::tmem_wait_st();
        float *mine = xb + ((r & 1) * 2 + half) * 4 * D;
        const float *other = xb + ((r & 1) * 2 + (1 - half)) * 4 * D;
        mine[j] = pv;
        mine[D + j] = pq;
        mine[2 * D + j] = kq;
        chain_bar();
        const float nk = kRaw ? nrm[C + r] : 1.f, nq = kRaw ? nrm[r] : 1.f;
        const float vh = (pv + other[j]) * nk;                  // S~^T k (unit key)
        const float ph = (pq + other[D + j]) * nq;              // S~^T q (unit query)
        const float kqs = (kq + other[2 * D + j]) * nk * nq;    // k . q
        const float vj = __bfloat162float(((const __nv_bfloat16 *)p.v)[row * D + j]);
        float e;
        if constexpr (kGate == kGateGdn2)   // e = w * v - S~^T (b * k)
            e = __bfloat162float(((const __nv_bfloat16 *)p.wgate)[row * D + j]) * vj - vh;
        else
            e = load_beta<kRaw>(p, sp, h, c, r) * (vj - vh);
        if (half == 0) st_elem(p.o, row * D + j, p.scale * fmaf(e, kqs, ph), p.out_bf16);
        const float ek = e * nk;
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            float sv[32];
            ptx::tmem_ld32(tcol + 32 * q2, sv);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float kv[8];
                ld_bf16x8(kr + 32 * q2 + 8 * g, kv);
#pragma unroll
                for (int i = 0; i < 8; ++i) sv[8 * g + i] = fmaf(kv[i], ek, sv[8 * g + i]);
            }
            ptx::tmem_st32(tcol + 32 * q2, sv);
        }
        ptx::tmem_wait_st();
    }
}

// Chain warps, a chunk that runs token by token (after its M3/M4 groups have completed;
// the E phase saved the chunk's initial state in the S' plane columns): put the state
// back into the fp32 state columns, run the tokens there, then write S'_{c+1}
// (unscaled when chunk c+1 also runs token by token) with its bf16 planes and clear the
// O accumulator, or store the final state.
template <int kGate, bool kRaw>
__device__ __forceinline__ void extreme_chunk(const ChunkArgs &p, uint8_t *sm, uint32_t tmem, uint32_t lane_base,
                                              const SeqSpan &sp, int h, int c, int half, int j, size_t tile,
                                              int nchunks, bool xn)
{
    const uint32_t tcol = tmem + lane_base + TM_S + 64 * half;
#pragma unroll 1
    for (int q2 = 0; q2 < 2; ++q2) {
        float v[32];
        ptx::tmem_ld32(tmem + lane_base + TM_SP + 64 * half + 32 * q2, v);
        ptx::tmem_wait_ld();
        ptx::tmem_st32(tcol + 32 * q2, v);
    }
    ptx::tmem_wait_st();
    // E^T is free until chunk c+1's readout: scratch for the two halves' sums.  The
    // barrier of the first token also orders every thread's read of the saved state
    // before the plane writes below.
    sequential_chunk<kGate, kRaw>(p, sm, tcol, sp, h, c, half, j, reinterpret_cast<float *>(sm + OFF_ET));
    if (c + 1 < nchunks) {
        const float *an = reinterpret_cast<const float *>(sm + OFF_CST + ((c + 1) % kCstSlots) * CST_BYTES);
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half);
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half + 16);
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
            const int d0 = 64 * half + 16 * part;
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + TM_S + d0, v);
            ptx::tmem_wait_ld();
            write_state16(tmem, lane_base, d0, v, an + d0, xn);
        }
        ptx::tmem_wait_st();
    } else if (p.s_out) {
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
            const int d0 = 64 * half + 16 * part;
            float v[16];
            ptx::tmem_ld16(tmem + lane_base + TM_S + d0, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) p.s_out[tile + (size_t)(d0 + i) * D + j] = v[i];
        }
    }
}

// ---- the chain warps: the serial recurrence over chunks --------------------------------
template <int kGate, bool kRaw, bool kLateB>
__device__ void chain_role(const ChunkArgs &p, const TcMaps &maps, uint8_t *sm, uint32_t tmem, const Bars &bars,
                           const TmaPos &tp, const SeqSpan &sp, int h, int bh, int nchunks, volatile int *err_flag)
{
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int j = quad * 32 + lane;            // value channel = TMEM lane
    const size_t tile = (size_t)bh * D * D;

    uint32_t ie[16];   // R of the chunk being staged (split words), carried from part A to part B
    if (tid == kTmaThread) {
        load_qka<kGate>(maps, sm, bars, tp, 0);
        for (int n = 1; n < 4 && n < nchunks; ++n) prefetch_qka<kGate>(maps, tp, n);
    }
    int staged = 0;   // chunks whose rows have been waited for
    chain_stage_a<kGate, kRaw>(p, sm, bars, sp, h, 0, warp, lane, ie, err_flag);
    staged = 1;
    chain_stage_b<kGate>(maps, sm, bars, tp, 0, nchunks, tid, warp, lane, ie);

    // S'_0 = Diag(exp(a_0)) S_0 (S_0 itself when chunk 0 runs token by token); cleared O
    {
        const float *cst0 = reinterpret_cast<const float *>(sm + OFF_CST);
        const bool x0 = chunk_is_extreme(sm, 0);
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
            const int d0 = 64 * half + 16 * part;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = p.s_in ? p.s_in[tile + (size_t)(d0 + i) * D + j] : 0.f;
            write_state16(tmem, lane_base, d0, v, cst0 + d0, x0);
        }
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half);
        ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half + 16);
        ptx::tmem_wait_st();
    }
    ptx::tc_fence_before();
    warp_signal(bars.rs, lane);
    if (nchunks > 1) {
        chain_stage_a<kGate, kRaw>(p, sm, bars, sp, h, 1, warp, lane, ie, err_flag);
        staged = 2;
        chain_stage_b<kGate>(maps, sm, bars, tp, 1, nchunks, tid, warp, lane, ie);
    }

    for (int c = 0; c < nchunks; ++c) {
        // the rows of chunk c+4 into L2: their staging load (issued at the end of
        // iteration c+1) then does not wait for HBM
        if (tid == kTmaThread && c + 4 < nchunks) prefetch_qka<kGate>(maps, tp, c + 4);
        // ---- E: E^T = U^T - S'^T W'^T (hi and lo column groups) into the A operand of M4
        if (!ptx::mbar_wait(bars.e, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        const bool xc = chunk_is_extreme(sm, c);
        if (xc) {
            // the chunk runs token by token: keep its initial state (unscaled, written so by
            // the previous chunk's rewrite) in the S' plane columns, which M3 has finished
            // reading; the state update of M4 then changes nothing that is used
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                float v[32];
                ptx::tmem_ld32(tmem + lane_base + TM_S + 64 * half + 32 * q2, v);
                ptx::tmem_wait_ld();
                ptx::tmem_st32(tmem + lane_base + TM_SP + 64 * half + 32 * q2, v);
            }
            ptx::tmem_wait_st();
        } else {
            // token blocks 2 half and 2 half + 1, each as [hi 8 | lo 8] columns
            float v0[16], v1[16];
            ptx::tmem_ld16(tmem + lane_base + TM_E + 32 * half, v0);
            ptx::tmem_ld16(tmem + lane_base + TM_E + 32 * half + 16, v1);
            ptx::tmem_wait_ld();
            float e0[8], e1[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                e0[i] = v0[i] + v0[8 + i];
                e1[i] = v1[i] + v1[8 + i];
            }
            if constexpr (kRaw) {   // the operand is Diag(nk) E (tokens 16 half + i, 16 half + 8 + i)
                const float *nk = reinterpret_cast<const float *>(sm + OFF_NRM + (c % kNrmSlots) * NRM_BYTES) + C;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    e0[i] *= nk[16 * half + i];
                    e1[i] *= nk[16 * half + 8 + i];
                }
            }
            st_split8(sm + OFF_ET + ipl(j, 16 * half, 0), C * 16, e0);
            st_split8(sm + OFF_ET + ipl(j, 16 * half + 8, 0), C * 16, e1);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        warp_signal(bars.re, lane);
        // Lk, Lq of chunk c+2 while the state update of chunk c runs
        if (c + 2 < nchunks) {
            chain_stage_a<kGate, kRaw>(p, sm, bars, sp, h, c + 2, warp, lane, ie, err_flag);
            staged = c + 3;
        }

        // ---- I: X = S' + E^T R -> the next S' (or the final state); outputs of chunk c
        if (!ptx::mbar_wait(bars.s, (uint32_t)(c & 1), kWaitLimitNs)) *err_flag = 1;
        ptx::tc_fence_after();
        const bool xn = c + 1 < nchunks && chunk_is_extreme(sm, c + 1);
        // R of chunk c+2 (the update of chunk c has read R(c)): here, or (kLateB) after the
        // state rewrite below, which is on the chain -- measured faster when the grid has
        // more blocks than half the SMs, slower when it has fewer; before a token-by-token
        // chunk always here
        if ((xc || !kLateB) && c + 2 < nchunks) {
            stage_b(sm, c + 2, warp, lane, ie);
            warp_signal_after_stage(bars, c + 2, lane);
        }
        if (xc) {
            // outputs stored token by token; the staging rows (read by every warp's stage A
            // above, and by the previous chunk's output store) are then free for chunk c+3
            extreme_chunk<kGate, kRaw>(p, sm, tmem, lane_base, sp, h, c, half, j, tile, nchunks, xn);
            if (c + 1 < nchunks) {
                ptx::tc_fence_before();
                warp_signal(bars.rs, lane);
            }
            const bool stop = chain_bar_err(err_flag);
            if (tid == kTmaThread && c + 3 < nchunks) {
                ptx::bulk_wait_read();
                load_qka<kGate>(maps, sm, bars, tp, c + 3);
            }
            if (stop) break;
            continue;
        }
        float ov[16];
        {
            float v0[16], v1[16];
            ptx::tmem_ld16(tmem + lane_base + TM_O + 32 * half, v0);
            ptx::tmem_ld16(tmem + lane_base + TM_O + 32 * half + 16, v1);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ov[i] = v0[i] + v0[8 + i];
                ov[8 + i] = v1[i] + v1[8 + i];
            }
            if constexpr (kRaw) {   // O -> Diag(nq) O
                const float *nq = reinterpret_cast<const float *>(sm + OFF_NRM + (c % kNrmSlots) * NRM_BYTES);
#pragma unroll
                for (int i = 0; i < 16; ++i) ov[i] *= nq[16 * half + i];
            }
        }
        if (c + 1 < nchunks) {
            // f(c+1) = exp(a_{c+1}) exp(G_end,c - a_c), written when chunk c+1 was staged; when
            // chunk c+1 runs token by token its initial state is kept unscaled: exp(G_end,c - a_c)
            const float *f = xn ? reinterpret_cast<const float *>(sm + OFF_CST + (c % kCstSlots) * CST_BYTES) + D
                                : reinterpret_cast<const float *>(sm + OFF_CST + ((c + 1) % kCstSlots) * CST_BYTES) + 2 * D;
            ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half);
            ptx::tmem_st16_zero(tmem + lane_base + TM_O + 32 * half + 16);
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                const int d0 = 64 * half + 32 * q2;
                float v[32];
                ptx::tmem_ld32(tmem + lane_base + TM_S + d0, v);
                ptx::tmem_wait_ld();
                const float4 *f4 = reinterpret_cast<const float4 *>(f + d0);
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    const float4 ff = f4[i4];
                    ptx::upk2(ptx::mul2(ptx::pk2(v[4 * i4], v[4 * i4 + 1]), ptx::pk2(ff.x, ff.y)), v[4 * i4],
                              v[4 * i4 + 1]);
                    ptx::upk2(ptx::mul2(ptx::pk2(v[4 * i4 + 2], v[4 * i4 + 3]), ptx::pk2(ff.z, ff.w)), v[4 * i4 + 2],
                              v[4 * i4 + 3]);
                }
                ptx::tmem_st32(tmem + lane_base + TM_S + d0, v);
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) split_pair(v[2 * m], v[2 * m + 1], hw[m], lw[m]);
                ptx::tmem_st16(tmem + lane_base + TM_SP + d0 / 2, hw);
                ptx::tmem_st16(tmem + lane_base + TM_SP + 64 + d0 / 2, lw);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            warp_signal(bars.rs, lane);
            if (kLateB && c + 2 < nchunks) {   // R of chunk c+2, once S' is out
                stage_b(sm, c + 2, warp, lane, ie);
                warp_signal_after_stage(bars, c + 2, lane);
            }
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
        // outputs of chunk c into the staging rows q and alpha have left (rows 16h..16h+15
        // into the q rows for h = 0, the alpha rows for h = 1), as one TMA box each.
        // Those rows still hold chunk c+2's q, k and alpha until every chain warp has
        // finished its stage A of chunk c+2, so the tile is written only after a chain
        // barrier.  The previous chunk's output store must also have read the rows: a
        // staging fill orders that (thread 0 issues it after the read); without one,
        // thread 0 waits for the read here, before the barrier.
        if (c > 0 && c + 2 >= nchunks && tid == kTmaThread) ptx::bulk_wait_read();
        chain_bar();
        const bool full = (c + 1) * C <= sp.len;
        if (full) {
            const int esz = p.out_bf16 ? 2 : 4;
            uint8_t *otile = sm + OFF_STG + (half ? STG_A : STG_Q) + j * esz;
            if (p.out_bf16) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    *reinterpret_cast<__nv_bfloat16 *>(otile + i * D * 2) = __float2bfloat16_rn(ov[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) *reinterpret_cast<float *>(otile + i * D * 4) = ov[i];
            }
        } else {
            // the sequence's last, partial chunk: only its own rows, one element per row
            // (a TMA box would also cover rows that belong to the next sequence)
            const size_t step = (size_t)p.H * D;
            size_t idx = ((sp.tok0 + (size_t)c * C + 16 * half) * p.H + h) * D + j;
#pragma unroll
            for (int i = 0; i < 16; ++i, idx += step)
                if (c * C + 16 * half + i < sp.len) st_elem(p.o, idx, ov[i], p.out_bf16);
        }
        ptx::fence_proxy_async_smem();
        const bool stop = chain_bar_err(err_flag);   // output tile written, staging rows consumed
        if (tid == kTmaThread) {
            if (full) {
                ptx::tma_store_4d(&maps.o, ptx::smem_u32(sm + OFF_STG + STG_Q), 0, h, tp.t0 + c * C, tp.b);
                ptx::tma_store_4d(&maps.o, ptx::smem_u32(sm + OFF_STG + STG_A), 0, h, tp.t0 + c * C + 16, tp.b);
            }
            ptx::bulk_commit();
            if (c + 3 < nchunks) {
                ptx::bulk_wait_read();   // the tile has been read: the staging rows can be refilled
                load_qka<kGate>(maps, sm, bars, tp, c + 3);
            }
        }
        if (stop) break;
    }
    // on an early exit, let a staging load still in flight land before the block ends
    if (staged < nchunks && staged > 0)
        (void)ptx::mbar_wait(bars.stg, (uint32_t)(staged & 1), kWaitLimitNs);
    if (tid == kTmaThread) ptx::bulk_wait();   // the output stores are complete
}

// kGate: alpha per key channel [B, T, H, d_k], or one retention factor per (token, head),
// alpha [B, T, H] (Gated DeltaNet), staged by TMA or read from memory.
// kRaw: the input preprocessing is fused into the kernel (raw q, k and logits).
template <int kGate, bool kRaw, bool kLateB>
__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(ChunkArgs pa, const __grid_constant__ TcMaps maps)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;                 // sequence * H + head (state tile)
    const int h = bh % pa.H;
    const ChunkArgs p = pa;
    SeqSpan sp;                                // the sequence's token rows
    if (!sequence_span(pa, bh / pa.H, sp)) {
        if (tid == 0 && pa.status) atomicOr(pa.status, 2u);
        return;
    }
    // TMA coordinates: dense tensors by (batch, token); packed ones as one batch by token row
    const TmaPos tp{pa.cu_seqlens ? 0 : bh / pa.H, h, pa.cu_seqlens ? (int)sp.tok0 : 0};
    const int nchunks = (sp.len + C - 1) / C;
    if (nchunks == 0) {
        // an empty sequence: the final state is the initial one (or zeros)
        if (p.s_out) {
            const size_t tile = (size_t)bh * D * D;
            for (int i = tid; i < D * D; i += NT) p.s_out[tile + i] = p.s_in ? p.s_in[tile + i] : 0.f;
        }
        return;
    }

    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *err_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    const uint32_t bar0 = ptx::smem_u32(sm + OFF_BAR);
    Bars bars;
    bars.a = bar0; bars.w = bar0 + 8; bars.e = bar0 + 16; bars.s = bar0 + 24;
    bars.stg = bar0 + 32; bars.v = bar0 + 40;   // v and v + 8
    bars.rc = bar0 + 56;   // and bar0 + 64
    bars.rs = bar0 + 72; bars.re = bar0 + 80;
    bars.ra = bar0 + 88; bars.rg = bar0 + 96; bars.rj = bar0 + 104;

    if (tid == 0) {
        ptx::mbar_init(bars.a, 1);
        ptx::mbar_init(bars.w, 1);
        ptx::mbar_init(bars.e, 1);
        ptx::mbar_init(bars.s, 1);
        ptx::mbar_init(bars.stg, 1);
        ptx::mbar_init(bars.v, 1);
        ptx::mbar_init(bars.v + 8, 1);
        ptx::mbar_init(bars.rc, NCW);
        ptx::mbar_init(bars.rc + 8, NCW);
        ptx::mbar_init(bars.rs, NCW);
        ptx::mbar_init(bars.re, NCW);
        ptx::mbar_init(bars.ra, NPW);
        ptx::mbar_init(bars.rg, NPW);
        ptx::mbar_init(bars.rj, NPW);
        ptx::fence_mbar_init();
#pragma unroll
        for (int i = 0; i < kXSlots; ++i) reinterpret_cast<int *>(sm + OFF_XF)[i] = 0;
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
        if (lane == 0) issuer<kGate, kRaw, kLateB>(sm, tmem, bars, nchunks, err_flag);
    } else if (warp >= NCW) {
        prep_role<kGate, kRaw>(p, maps, sm, tmem, bars, tp, sp, h, nchunks, err_flag);
    } else {
        chain_role<kGate, kRaw, kLateB>(p, maps, sm, tmem, bars, tp, sp, h, bh, nchunks, err_flag);
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

namespace {

// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time
// dependency on the driver library).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// q, k, alpha [B][T][H][128] bf16: dims (d, h, t, b), box (128, 1, 32, 1).
bool encode_rows(CUtensorMap *m, const void *base, int B, int T, int H)
{
    const cuuint64_t dims[4] = {(cuuint64_t)tc::D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)tc::D * 2, (cuuint64_t)H * tc::D * 2,
                                   (cuuint64_t)T * H * tc::D * 2};
    const cuuint32_t box[4] = {(cuuint32_t)tc::D, 1, (cuuint32_t)tc::C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// one gate per (token, head), [B][T][H] bf16: dims (h, t, b), box (8, 32, 1) -- 16-byte rows
bool encode_head_gate(CUtensorMap *m, const void *base, int B, int T, int H)
{
    const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)H * 2, (cuuint64_t)T * H * 2};
    const cuuint32_t box[3] = {8, (cuuint32_t)tc::C, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// v [B][T][H][128] bf16 as (j%8, t, j/8, h, b), box (8, 32, 16, 1, 1): the box lands
// as j/8-major, token-minor 16-byte rows, the MN-major core matrices of V^T.
bool encode_v(CUtensorMap *m, const void *base, int B, int T, int H)
{
    const cuuint64_t dims[5] = {8, (cuuint64_t)T, (cuuint64_t)tc::D / 8, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)H * tc::D * 2, 16, (cuuint64_t)tc::D * 2,
                                   (cuuint64_t)T * H * tc::D * 2};
    const cuuint32_t box[5] = {8, (cuuint32_t)tc::C, (cuuint32_t)tc::D / 8, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// o [B][T][H][128] fp32 or bf16: dims (j, h, t, b), box (128, 1, 16, 1).
bool encode_out(CUtensorMap *m, void *base, int B, int T, int H, int bf16)
{
    const cuuint64_t es = bf16 ? 2 : 4;
    const cuuint64_t dims[4] = {(cuuint64_t)tc::D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)tc::D * es, (cuuint64_t)H * tc::D * es, (cuuint64_t)T * H * tc::D * es};
    const cuuint32_t box[4] = {(cuuint32_t)tc::D, 1, 16, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_fn()(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const ChunkArgs &a, int dk, int dv, cudaStream_t stream)
{
    (void)dk; (void)dv;
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (encode_fn() == nullptr) return cudaErrorNotSupported;
    tc::TcMaps maps;
    const int mb = a.cu_seqlens ? 1 : a.B;   // packed sequences: one [1, T, H, d] tensor
    bool head_gate_tma = false;
    if (a.gate_per_head) {
        // [B][T][H] gates as boxes of 8 heads x 32 tokens when the layout allows a TMA box
        // (16-byte rows of heads and a 16-byte-aligned base); otherwise read per token
        memset(&maps.a, 0, sizeof(maps.a));
        head_gate_tma = a.H % 8 == 0 && ((uintptr_t)a.alpha & 15u) == 0 &&
                        encode_head_gate(&maps.a, a.alpha, mb, a.T, a.H);
    }
    const bool gdn2 = a.erase != nullptr;
    if (gdn2 && (!a.wgate || a.gate_per_head || a.raw_inputs)) return cudaErrorInvalidValue;
    memset(&maps.w, 0, sizeof(maps.w));
    memset(&maps.b, 0, sizeof(maps.b));
    if (gdn2 && (!encode_v(&maps.w, a.wgate, mb, a.T, a.H) || !encode_rows(&maps.b, a.erase, mb, a.T, a.H)))
        return cudaErrorInvalidValue;
    if (!encode_rows(&maps.q, a.q, mb, a.T, a.H) || !encode_rows(&maps.k, a.k, mb, a.T, a.H) ||
        (!a.gate_per_head && !encode_rows(&maps.a, a.alpha, mb, a.T, a.H)) || !encode_v(&maps.v, a.v, mb, a.T, a.H) ||
        !encode_out(&maps.o, a.o, mb, a.T, a.H, a.out_bf16))
        return cudaErrorInvalidValue;
    if (a.gate_per_head && a.raw_inputs) return cudaErrorInvalidValue;
    // The plain kernel stages R of the chunk two ahead after the state rewrite when the grid
    // fills more than half the SMs (prefill workload, 128 blocks: 2 % faster), before it
    // otherwise (long workload, 64 blocks: 3 % faster); the other gate kinds and the raw
    // inputs always before it (at 128 blocks the late form made them 3.4-5.5 % slower).
    // Measured on a B200, two builds timed alternately in one process.  A compile-time
    // choice: as a run-time flag the two placements in one kernel made the late one 3.5 %
    // slower.
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool late_b = 2 * blocks > sms;
    using tc::kda_chunk_tc_kernel;
    auto kernel = gdn2            ? kda_chunk_tc_kernel<tc::kGateGdn2, false, false>
                  : a.gate_per_head ? (head_gate_tma ? kda_chunk_tc_kernel<tc::kGateHeadTma, false, false>
                                                     : kda_chunk_tc_kernel<tc::kGateHeadMem, false, false>)
                  : a.raw_inputs    ? kda_chunk_tc_kernel<tc::kGateChannel, true, false>
                  : late_b          ? kda_chunk_tc_kernel<tc::kGateChannel, false, true>
                                    : kda_chunk_tc_kernel<tc::kGateChannel, false, false>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    kernel<<<(unsigned)blocks, tc::NT, tc::SMEM_BYTES, stream>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace kda
