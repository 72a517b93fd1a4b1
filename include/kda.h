/*
 * kda.h -- C ABI of the B200 (sm_100a) KDA library.
 *
 * KDA (Kimi Delta Attention) is the gated delta rule with one retention factor
 * per key channel.  For each (sequence, head), with a state S in R^{d_k x d_v}
 * (rows = key channels, columns = value channels) and per token t:
 *
 *   S~_t = Diag(alpha_t) S_{t-1}                 forget, per key channel
 *   vh_t = S~_t^T k_t                            predict
 *   e_t  = v_t - vh_t                            correct
 *   S_t  = S~_t + beta_t k_t e_t^T               write
 *   o_t  = S_t^T (scale q_t)                     read
 *
 * This is the five-step update of "Module 03 -- KDA I: The Delta-Rule
 * Recurrence" (jared-hpc.com), section 2, in the d_k x d_v layout of the
 * five-line recurrence in "Kimi Delta Attention (KDA)" (brain.bigb.es),
 * section "KDA: one gate per key channel"; the scale multiplies q at the read
 * only, as in that page's opening statement.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, row-major and contiguous, owned
 *    by the caller; the library allocates and frees nothing.
 *  - q, k, v, alpha, o and the state pointers must be 16-byte aligned; beta
 *    only needs its element alignment (KDA_ERR_ALIGN otherwise).
 *  - Argument errors are detected on the host and returned before anything
 *    is launched; nothing is written then.  Launch failures return
 *    KDA_ERR_LAUNCH.  Calls are asynchronous on `stream` (0 = legacy default
 *    stream); no call synchronizes.  No exception crosses the ABI.
 *  - Supported head sizes: d_k, d_v in {16, 32, 48, 64, 80, 96, 112, 128}
 *    (every multiple of 16 up to 128), in any combination; otherwise
 *    KDA_ERR_UNSUPPORTED.
 *  - alpha is the linear retention factor in (0, 1] (alpha = 0 is accepted and
 *    treated as a retention of e^-80 ~ 1.8e-35); beta is the write strength in
 *    [0, 1]; neither is range-checked.
 *  - Arithmetic and the state are fp32; bf16 inputs are read exactly.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of an input or output tensor. */
typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_NULL = 1,        /* a required pointer is NULL */
    KDA_ERR_SHAPE = 2,       /* a size is negative or a product overflows */
    KDA_ERR_DTYPE = 3,       /* unknown dtype code */
    KDA_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
    KDA_ERR_UNSUPPORTED = 5, /* head size not a multiple of 16 in [16, 128] */
    KDA_ERR_WORKSPACE = 6,   /* workspace too small or NULL when required */
    KDA_ERR_LAUNCH = 7,      /* the CUDA launch reported an error */
    KDA_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up */
    KDA_ERR_ALIAS = 9,       /* an output overlaps an input it must not alias */
    KDA_ERR_VALUE = 10       /* an enumerated argument has an unknown value */
} kda_status;

/*
 * Prefill schedule, process-wide (every prefill entry point that runs plain
 * KDA or the per-head gate: kda_forward, kda_forward_scalar_gate, the packed
 * kda_forward_varlen, their no-alloc and host-buffer forms).
 *   KDA_SCHEDULE_AUTO     (default) the tensor-core chunk kernel where it
 *                         applies (d_k = d_v = 128, bf16 inputs and gates),
 *                         otherwise the column scan (it is faster than the
 *                         CUDA-core chunk kernel at every size measured).
 *   KDA_SCHEDULE_CHUNKED  always the chunkwise schedule.
 *   KDA_SCHEDULE_SCAN     always the column scan where it applies.
 * The column scan is the token-by-token recurrence with every value column of
 * the state run as a chain of its own (column j of S depends only on k, q,
 * alpha, beta and v_j): "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two
 * schedules for the same recurrence", the fused recurrent form.  It does not
 * take raw inputs or GDN-2 gates; those always run chunkwise.  Both schedules
 * give the recurrence's result up to rounding.
 */
typedef enum { KDA_SCHEDULE_AUTO = 0, KDA_SCHEDULE_CHUNKED = 1, KDA_SCHEDULE_SCAN = 2 } kda_schedule;

/* Set the prefill schedule for later calls (KDA_ERR_VALUE for an unknown
 * value; the setting is then unchanged).  Affects calls made after it returns,
 * on any thread. */
kda_status kda_set_schedule(int schedule);

/* The current prefill schedule. */
int kda_get_schedule(void);

/*
 * kda_forward -- prefill: run the recurrence over T tokens for B sequences and
 * H heads with the chunkwise-parallel schedule on the tensor cores (d_k = d_v
 * = 128, bf16 inputs and gates), or with the column scan for other shapes and
 * dtypes (see kda_set_schedule).
 *
 * Defined by: "Kimi Delta Attention (KDA)" (brain.bigb.es), "Two schedules for
 * the same recurrence" (provisional errors, the unit-lower-triangular
 * correction, the one-shot state fast-forward and the diagonal-inclusive
 * read), and "From Fast Weight Programmers to KDA" (jonahsamost.bearblog.dev),
 * section "Kimi Delta Attention" (chunkwise WY/UT form with per-channel
 * cumulative decay).  The result equals the sequential recurrence above up to
 * rounding.
 *
 *   q, k, alpha   [B, T, H, d_k]   qkv_dtype (q, k) / gate_dtype (alpha)
 *   v             [B, T, H, d_v]   qkv_dtype
 *   beta          [B, T, H]        gate_dtype
 *   initial_state [B, H, d_k, d_v] fp32, may be NULL (zero state)
 *   o             [B, T, H, d_v]   out_dtype (written)
 *   final_state   [B, H, d_k, d_v] fp32, may be NULL (not returned); may be
 *                 the same pointer as initial_state (continuation in place)
 *   scale         multiplies q at the read (callers usually pass d_k^-1/2)
 *   workspace     device scratch of at least kda_forward_workspace_bytes()
 *                 bytes, 16-byte aligned, owned by the caller.  The call
 *                 zeroes it on `stream` and the kernel records there whether a
 *                 bounded device-side wait gave up; read it with
 *                 kda_workspace_status().  Calls that share a workspace must
 *                 not overlap on the GPU.
 * T = 0 copies initial_state (or zeros) to final_state.  o must not overlap
 * any input (KDA_ERR_ALIAS).  A last chunk shorter than the chunk size is
 * handled exactly (no padding of the caller's buffers is needed).
 */
kda_status kda_forward(const void *q, const void *k, const void *v,
                       const void *alpha, const void *beta,
                       const float *initial_state, void *o, float *final_state,
                       int B, int T, int H, int d_k, int d_v, float scale,
                       kda_dtype qkv_dtype, kda_dtype gate_dtype,
                       kda_dtype out_dtype, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/* Bytes of device workspace kda_forward needs for these sizes (currently 16:
 * one status word and padding, independent of the sizes). */
size_t kda_forward_workspace_bytes(int B, int T, int H, int d_k, int d_v);

/*
 * kda_workspace_status -- synchronize `stream`, then read the status word a
 * kda_forward or kda_forward_varlen call left in `workspace`: KDA_OK,
 * KDA_ERR_SHAPE when kda_forward_varlen met invalid sequence offsets, or
 * KDA_ERR_TIMEOUT when one of the kernel's bounded waits on its own tensor-core
 * completions gave up (the outputs of that call are then not valid).  KDA_ERR_LAUNCH if the copy or the
 * synchronization fails.  Not part of the recurrence; the pages have no
 * counterpart.
 */
kda_status kda_workspace_status(const void *workspace, cudaStream_t stream);

/*
 * kda_forward_noalloc -- kda_forward for callers that cannot allocate device
 * memory (an allocator-less runtime, a plugin that must not touch its host's
 * memory pool, code without an allocation API at hand).  Same arguments and
 * results as kda_forward, without the workspace: the library uses its own
 * fixed device array of 256 bytes (held on every GPU that loads the library
 * until the process exits) and returns KDA_ERR_WORKSPACE if a call would need
 * more than that.  Nothing is allocated or freed.  Every call shares that
 * array and clears it at its start, so calls that overlap on the GPU race:
 * serialize them.  The first call on a device looks up the array's address
 * (once per device, with that device current); make it before any stream
 * capture.  The kernel's status word (a bounded wait that gave up) lands in that
 * array, not in a caller's workspace: read it with kda_noalloc_status().  The
 * pages have no counterpart of this entry point.
 */
kda_status kda_forward_noalloc(const void *q, const void *k, const void *v,
                               const void *alpha, const void *beta,
                               const float *initial_state, void *o,
                               float *final_state, int B, int T, int H,
                               int d_k, int d_v, float scale,
                               kda_dtype qkv_dtype, kda_dtype gate_dtype,
                               kda_dtype out_dtype, cudaStream_t stream);

/*
 * kda_noalloc_status -- synchronize `stream`, then read the status word that
 * the last kda_forward_noalloc call on the current device left in the
 * library's array: KDA_OK, or KDA_ERR_TIMEOUT when one of the kernel's bounded
 * waits gave up (that call's outputs are then not valid); KDA_ERR_LAUNCH if
 * the array cannot be reached or the read fails.  Allocates nothing.  Call it
 * before the next kda_forward_noalloc on the device (each call clears the
 * word).  Like kda_forward_noalloc, no counterpart on the pages.
 */
kda_status kda_noalloc_status(cudaStream_t stream);

/*
 * kda_forward_varlen -- kda_forward over a packed batch of N sequences of
 * different lengths (the serving layout: no padding between sequences).
 * Sequence b owns token rows cu_seqlens[b] .. cu_seqlens[b+1]-1; each runs the
 * recurrence from its own initial state.  Defined by the same passages as
 * kda_forward.  The state of each sequence is per-request serving state
 * ("Module 03 -- KDA I: The Delta-Rule Recurrence", jared-hpc.com, section 5,
 * "State vs. checkpoint weights"); packing requests of different lengths into
 * one launch is a serving layout, not part of the recurrence.
 *
 *   q, k, alpha   [total_T, H, d_k]  (a [1, total_T, H, d_k] batch)
 *   v, o          [total_T, H, d_v]
 *   beta          [total_T, H]
 *   cu_seqlens    DEVICE int32 [N + 1]: 0 = cu_seqlens[0] <= ... <=
 *                 cu_seqlens[N] <= total_T, 4-byte aligned, owned by the caller
 *   initial_state [N, H, d_k, d_v] fp32 or NULL; final_state [N, H, d_k, d_v]
 *                 fp32 or NULL (may equal initial_state)
 * Other arguments as kda_forward.  The offsets live on the device, so they
 * are checked by the kernel: a sequence whose offsets are out of order or out
 * of range is skipped (nothing of it is written) and kda_workspace_status()
 * then returns KDA_ERR_SHAPE.  An empty sequence copies its initial state (or
 * zeros) to its final state.  Rows of o outside every sequence are not written.
 */
kda_status kda_forward_varlen(const void *q, const void *k, const void *v,
                              const void *alpha, const void *beta,
                              const int *cu_seqlens, const float *initial_state,
                              void *o, float *final_state, int N, int total_T,
                              int H, int d_k, int d_v, float scale,
                              kda_dtype qkv_dtype, kda_dtype gate_dtype,
                              kda_dtype out_dtype, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_forward_varlen_raw -- kda_forward_varlen on raw inputs: the preprocessing of
 * kda_forward_raw (q, k divided by their row norms in the kernel, gate logits
 * [total_T, H, d_k] with alpha = 1 / (1 + e^x), beta logits [total_T, H] with beta =
 * sigmoid(y)) over packed sequences.  Other arguments, layouts and errors as
 * kda_forward_varlen.
 */
kda_status kda_forward_varlen_raw(const void *q, const void *k, const void *v,
                                  const void *gate_logit, const void *beta_logit,
                                  const int *cu_seqlens, const float *initial_state,
                                  void *o, float *final_state, int N, int total_T,
                                  int H, int d_k, int d_v, float scale,
                                  kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                  kda_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_forward_varlen_gdn2 -- kda_forward_gdn2 over packed sequences: erase [total_T, H,
 * d_k] and write [total_T, H, d_v] gates (16-byte aligned) in place of beta.  Other
 * arguments, layouts and errors as kda_forward_varlen.
 */
kda_status kda_forward_varlen_gdn2(const void *q, const void *k, const void *v,
                                   const void *alpha, const void *erase,
                                   const void *write, const int *cu_seqlens,
                                   const float *initial_state, void *o,
                                   float *final_state, int N, int total_T, int H,
                                   int d_k, int d_v, float scale,
                                   kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                   kda_dtype out_dtype, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_forward_scalar_gate -- kda_forward with one retention factor per (token,
 * head): Gated DeltaNet, S~_t = alpha_t S_{t-1} with a scalar alpha_t, which is
 * KDA with alpha_t broadcast over the key channels ("From Fast Weight
 * Programmers to KDA", jonahsamost.bearblog.dev, section "Gated Delta
 * Networks"; "Notes on Linear Attention: From Linear Attention to KDA",
 * zhilingong.com, section 6 "Why add a gate?").  Arguments as
 * kda_forward except alpha, which is [B, T, H] (gate_dtype, element-aligned
 * like beta).  The per-channel decay work becomes per-token, and alpha's bytes
 * shrink by d_k.
 */
kda_status kda_forward_scalar_gate(const void *q, const void *k, const void *v,
                                   const void *alpha, const void *beta,
                                   const float *initial_state, void *o,
                                   float *final_state, int B, int T, int H,
                                   int d_k, int d_v, float scale,
                                   kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                   kda_dtype out_dtype, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_forward_gdn2 -- prefill of GDN-2, the gated delta rule with decoupled
 * gates ("From Fast Weight Programmers to KDA", jonahsamost.bearblog.dev,
 * section "Gated DeltaNet-2"): beta_t is replaced by an erase gate b_t (one
 * per key channel) and a write gate w_t (one per value channel):
 *
 *   S~_t = Diag(alpha_t) S_{t-1},  vh_t = S~_t^T (b_t * k_t),
 *   S_t  = S~_t + k_t (w_t * v_t - vh_t)^T,  o_t = S_t^T (scale q_t)
 *
 * (* elementwise; that page writes the state transposed).  b_t = beta_t 1 and
 * w_t = beta_t 1 give kda_forward.  Arguments as kda_forward with
 *   erase [B, T, H, d_k] and write [B, T, H, d_v]  (gate_dtype, 16-byte
 *   aligned) in place of beta.
 * Computed by the chunkwise schedule on the tensor cores for d_k = d_v = 128 with
 * bf16 inputs and gates, on CUDA cores in fp32 for every other supported shape and
 * dtype.
 */
kda_status kda_forward_gdn2(const void *q, const void *k, const void *v,
                            const void *alpha, const void *erase,
                            const void *write, const float *initial_state,
                            void *o, float *final_state, int B, int T, int H,
                            int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                            kda_dtype gate_dtype, kda_dtype out_dtype,
                            void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * kda_forward_sequential -- the same operation and arguments as kda_forward
 * (no workspace), computed with the token-by-token schedule ("fused
 * recurrent" in "Two schedules for the same recurrence", brain.bigb.es): one
 * block per (sequence, head) keeps its state on chip and walks the tokens in
 * order.  It exists so the two schedules can be checked against each other on
 * the GPU; it is not the fast path for long T.
 */
kda_status kda_forward_sequential(const void *q, const void *k, const void *v,
                                  const void *alpha, const void *beta,
                                  const float *initial_state, void *o,
                                  float *final_state, int B, int T, int H,
                                  int d_k, int d_v, float scale,
                                  kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                  kda_dtype out_dtype, cudaStream_t stream);

/*
 * kda_decode_step -- one token for each of N independent sequences, state
 * updated in place: the five-step update of "Module 03", section 2, once.
 * Each fp32 state tile is read from HBM once and written once; both
 * reductions (S~^T k and S~^T q) come from the same read, using
 * o = scale (S~^T q + e (k . q)) with e = beta (v - S~^T k).
 *
 *   q, k, alpha [N, H, d_k]  v [N, H, d_v]  beta [N, H]
 *   state       [N, H, d_k, d_v] fp32, read and overwritten
 *   o           [N, H, d_v] out_dtype (must not overlap state or inputs)
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *alpha, const void *beta, float *state,
                           void *o, int N, int H, int d_k, int d_v, float scale,
                           kda_dtype qkv_dtype, kda_dtype gate_dtype,
                           kda_dtype out_dtype, cudaStream_t stream);

/*
 * kda_decode_step_scalar_gate -- kda_decode_step with one retention factor per
 * (sequence, head): alpha is [N, H] (gate_dtype, element-aligned), broadcast
 * over the key channels (Gated DeltaNet; see kda_forward_scalar_gate).
 */
kda_status kda_decode_step_scalar_gate(const void *q, const void *k,
                                       const void *v, const void *alpha,
                                       const void *beta, float *state, void *o,
                                       int N, int H, int d_k, int d_v,
                                       float scale, kda_dtype qkv_dtype,
                                       kda_dtype gate_dtype,
                                       kda_dtype out_dtype,
                                       cudaStream_t stream);

/*
 * kda_forward_raw -- kda_forward with the input preprocessing fused into the
 * kernels' load stage, so that no separate pass over the inputs is needed:
 *   q, k        un-normalised projections; each token's q_t and k_t are
 *               divided by their L2 norms in the kernel (a zero row stays
 *               zero) -- "Notes on Linear Attention: From Linear Attention to
 *               KDA", section 5.3 "Why L2-normalize the key?" (and the
 *               query likewise, section 3)
 *   gate_logit  [B, T, H, d_k] gate_dtype: x with log alpha = -softplus(x),
 *               i.e. alpha = 1 / (1 + e^x) -- the stored log-decay
 *               g = log alpha <= 0 of "Kimi Delta Attention (KDA)"
 *               (brain.bigb.es), in the exp(-softplus) form of the gate
 *   beta_logit  [B, T, H] gate_dtype: y with beta = sigmoid(y) ("From Fast
 *               Weight Programmers to KDA", the delta rule's write strength)
 * Everything else (layouts, workspace, aliasing, status) is as kda_forward.
 */
kda_status kda_forward_raw(const void *q, const void *k, const void *v,
                           const void *gate_logit, const void *beta_logit,
                           const float *initial_state, void *o,
                           float *final_state, int B, int T, int H, int d_k,
                           int d_v, float scale, kda_dtype qkv_dtype,
                           kda_dtype gate_dtype, kda_dtype out_dtype,
                           void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * kda_decode_step_raw -- kda_decode_step on raw inputs (the preprocessing of
 * kda_forward_raw): q, k [N, H, d_k] un-normalised, gate_logit [N, H, d_k],
 * beta_logit [N, H]; the state [N, H, d_k, d_v] is updated in place.
 */
kda_status kda_decode_step_raw(const void *q, const void *k, const void *v,
                               const void *gate_logit, const void *beta_logit,
                               float *state, void *o, int N, int H, int d_k,
                               int d_v, float scale, kda_dtype qkv_dtype,
                               kda_dtype gate_dtype, kda_dtype out_dtype,
                               cudaStream_t stream);

/*
 * kda_decode_step_gdn2 -- kda_decode_step for GDN-2 (see kda_forward_gdn2):
 * erase [N, H, d_k] and write [N, H, d_v] (gate_dtype, 16-byte aligned) in
 * place of beta; the state [N, H, d_k, d_v] is updated in place.
 */
kda_status kda_decode_step_gdn2(const void *q, const void *k, const void *v,
                                const void *alpha, const void *erase,
                                const void *write, float *state, void *o,
                                int N, int H, int d_k, int d_v, float scale,
                                kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                kda_dtype out_dtype, cudaStream_t stream);

/*
 * Host-buffer entry points: for a caller whose tensors live in host memory (pinned
 * memory lets the copies overlap the kernels; pageable memory works but copies
 * synchronously).  The library copies the inputs in and the results out itself; not
 * part of the recurrence, and the pages have no counterpart.
 *
 * kda_forward_host -- one prefill (kind KDA_HOST_FORWARD: kda_forward;
 * KDA_HOST_SCALAR_GATE: kda_forward_scalar_gate, alpha [B, T, H]; KDA_HOST_RAW:
 * kda_forward_raw) with q, k, v, alpha, beta, initial_state (or NULL), o and
 * final_state (or NULL) all HOST pointers in the layouts of those entry points.
 * The sequence is cut into segments of 1024 tokens: segment j+1 is copied in on an
 * internal stream while the kernel runs segment j on `stream`, continuing from
 * segment j-1's state, and segment j-1's outputs are copied back on another internal
 * stream.  workspace: DEVICE memory of kda_forward_host_workspace_bytes() bytes,
 * 256-byte aligned, owned by the caller: two slots of segment buffers, the carried
 * state and, at offset 0, the status word (read it with kda_workspace_status()).
 * Asynchronous: everything is ordered after the work already on `stream`, and work
 * queued on `stream` afterwards (a synchronization included) starts only once the
 * last result is back in host memory.  The host buffers must stay valid until then.
 * Argument errors return before anything is queued; a failing segment returns its
 * status (work already queued still runs).
 */
typedef enum { KDA_HOST_FORWARD = 0, KDA_HOST_SCALAR_GATE = 1, KDA_HOST_RAW = 2 } kda_host_kind;

size_t kda_forward_host_workspace_bytes(int B, int T, int H, int d_k, int d_v,
                                        kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                        kda_dtype out_dtype, int kind);

kda_status kda_forward_host(int kind, const void *q, const void *k,
                            const void *v, const void *alpha, const void *beta,
                            const float *initial_state, void *o,
                            float *final_state, int B, int T, int H, int d_k,
                            int d_v, float scale, kda_dtype qkv_dtype,
                            kda_dtype gate_dtype, kda_dtype out_dtype,
                            void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * kda_decode_step_host -- kda_decode_step with q, k, alpha [N, H, d_k], v [N, H, d_v],
 * beta [N, H] and o [N, H, d_v] in HOST memory, and the state [N, H, d_k, d_v] fp32 in
 * DEVICE memory (it stays resident between steps, like a KV cache), updated in place.
 * The copies and the kernel run in order on `stream`; workspace: DEVICE memory of
 * kda_decode_step_host_workspace_bytes() bytes, 256-byte aligned, for the token
 * vectors and o.  Asynchronous like kda_forward_host.
 */
size_t kda_decode_step_host_workspace_bytes(int N, int H, int d_k, int d_v,
                                            kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                            kda_dtype out_dtype);

kda_status kda_decode_step_host(const void *q, const void *k, const void *v,
                                const void *alpha, const void *beta, float *state,
                                void *o, int N, int H, int d_k, int d_v, float scale,
                                kda_dtype qkv_dtype, kda_dtype gate_dtype,
                                kda_dtype out_dtype, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/*
 * Serving operations.  A recurrent state is request-scoped, like a KV-cache
 * slot: it is cached between turns and must be copied whenever a request is
 * forked, shares a prefix, migrates or is rolled back after a speculative
 * step ("Module 03 -- KDA I: The Delta-Rule Recurrence", section 5 "State vs.
 * checkpoint weights").  States live in pools of slots [slots, H, d_k, d_v]
 * fp32.
 *
 * kda_decode_tokens -- T tokens per sequence through the recurrence of
 * kda_decode_step, token after token (the draft tokens of a speculative step;
 * T = 1 is a plain decode step over a slot pool).
 *   q, k, alpha   [N, T, H, d_k]   v [N, T, H, d_v]   beta [N, T, H]
 *   o             [N, T, H, d_v]   out_dtype (written)
 *   state         pool [num_slots, H, d_k, d_v] fp32; sequence n starts from
 *                 slot state_slots[n] (slot n when state_slots is NULL, then
 *                 num_slots >= N is required).  A negative slot skips the
 *                 sequence (its rows of o are not written); a slot >=
 *                 num_slots is skipped too and recorded in the status word.
 *   commit        nonzero: the state after the T tokens is written back to the
 *                 sequence's slot; zero: the pool is only read (verification).
 *   token_states  [N, T, H, d_k, d_v] fp32 or NULL: the state after each
 *                 token, so that a rejected suffix can be rolled back with
 *                 kda_state_copy (accepted prefix of a_n >= 1 tokens: source
 *                 index n*T + a_n - 1 of token_states viewed as N*T slots).
 *   status        NULL or a 16-byte-aligned device word (for instance a
 *                 workspace of kda_forward_workspace_bytes() bytes), zeroed
 *                 by the call; read it with kda_workspace_status()
 *                 (KDA_ERR_SHAPE: a slot index was out of range).
 * Two sequences must not name the same slot when commit is set.  o, the pool
 * and token_states must not overlap (KDA_ERR_ALIAS).
 */
kda_status kda_decode_tokens(const void *q, const void *k, const void *v,
                             const void *alpha, const void *beta, float *state,
                             const int *state_slots, int num_slots, int commit,
                             float *token_states, void *o, int N, int T, int H,
                             int d_k, int d_v, float scale, kda_dtype qkv_dtype,
                             kda_dtype gate_dtype, kda_dtype out_dtype,
                             void *status, cudaStream_t stream);

/*
 * kda_state_copy -- entry i (i < count) copies the state block
 * src[src_index[i]] to dst[dst_index[i]], each block [H, d_k, d_v] fp32.
 *   src, dst      pools of src_slots and dst_slots blocks (may be the same
 *                 pool: a fork inside one pool)
 *   src_index, dst_index  [count] int32 on the device, or NULL for the
 *                 identity index i (then count may not exceed that pool's
 *                 slots).  An entry with a negative index is skipped; one with
 *                 an index past its pool is skipped and recorded in the status
 *                 word (KDA_ERR_SHAPE from kda_workspace_status()).
 *   status        as for kda_decode_tokens.
 * A block that one entry writes must not be read or written by another entry
 * of the same call.  The copy is asynchronous on `stream`.
 */
kda_status kda_state_copy(const float *src, const int *src_index, int src_slots,
                          float *dst, const int *dst_index, int dst_slots,
                          int count, int H, int d_k, int d_v, void *status,
                          cudaStream_t stream);

/*
 * kda_selftest_bounded_wait -- a check of the device-side failure detection that
 * the tensor-core prefill uses (no counterpart on the pages): one thread waits on an
 * mbarrier with the prefill's bounded-wait helper.  arrive != 0 completes the
 * barrier's phase first (the wait succeeds); arrive == 0 leaves it incomplete, so
 * the wait gives up after limit_us microseconds (1 .. 2,000,000) and records the
 * timeout in the status word.  status: a 16-byte-aligned device word (for instance a
 * workspace of kda_forward_workspace_bytes() bytes), zeroed by the call; read it with
 * kda_workspace_status(): KDA_ERR_TIMEOUT after a wait that gave up, KDA_OK
 * otherwise.  The kernel returns normally either way; the context stays usable.
 */
kda_status kda_selftest_bounded_wait(int arrive, unsigned int limit_us, void *status,
                                     cudaStream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *kda_status_string(kda_status status);

/* Library version as 10000*major + 100*minor + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H */
