/*
 * lmoe.h -- C ABI of the B200 (sm_100a) LatentMoE layer forward pass.
 *
 * The layer (LatentMoE: Toward Optimal Accuracy per FLOP and Parameter in
 * Mixture of Experts, arXiv 2601.18089, Section 3, Eq. (1) and Eq. (2)):
 *
 *   logits = x Wg (+ bias)                     router, full width d
 *   slots  = top-k of logits, ties to the lowest expert index
 *   w      = softmax over the k selected logits (renormalised gates)
 *   z      = x Wdown                           down-projection d -> l
 *   y_j    = act(z W1[e_j]) W2[e_j]            routed experts in latent width
 *   comb   = sum_j w_j y_j                     gate-weighted combine
 *   out    = x + comb Wup + act(x Ws1) Ws2     up-projection, shared expert,
 *                                              residual add
 *
 * act is SiLU (non-gated), SwiGLU (FC1 has 2m columns: [0,m) is the SiLU
 * gate, [m,2m) the linear half) or squared ReLU (non-gated).  The shared
 * expert, when present, uses the same act.  With LMOE_SKIP_PROJ the layer is
 * the paper's standard MoE (Table 1, first row): l == d, z = x, u = comb.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the handle's device, row
 *     major and contiguous, unless a parameter says "host".  The caller owns
 *     them; the library never frees or retains them past the call.
 *   - Weights use the API layout [in, out] (y = x W).
 *   - dtype (set at create) applies to x, out and every weight; the router
 *     bias and all logits are fp32; indices are int32.
 *   - Calls taking a stream are asynchronous on it: they enqueue work and
 *     return; results are ready when the stream is.  They never allocate and
 *     never synchronise the host, except where stated.
 *   - Errors are returned as lmoe_status and never thrown.  Arguments are
 *     validated before any work is enqueued; on an error nothing is enqueued.
 *     Device-side failures (a bounded wait that ran out, a failed debug
 *     check) set a device error word that lmoe_last_error reads.
 *   - A handle is not thread safe: one host thread at a time per handle.
 *     Calls on one handle share its workspace, so calls enqueued on
 *     different streams must not overlap on the GPU.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* lmoe_stream_t;

typedef enum {
  LMOE_OK = 0,
  LMOE_ERR_INVALID_ARG = 1,   /* a bad size, pointer, flag or state         */
  LMOE_ERR_NOT_READY = 2,     /* weights not set / workspace not reserved   */
  LMOE_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed       */
  LMOE_ERR_OOM = 4,           /* device allocation failed                   */
  LMOE_ERR_TIMEOUT = 5,       /* a device-side bounded wait gave up         */
  LMOE_ERR_UNSUPPORTED = 6,   /* valid but outside the library's limits     */
  LMOE_ERR_DEVICE = 7         /* a device-side check failed (error word)    */
} lmoe_status;

typedef enum { LMOE_ACT_SILU = 0, LMOE_ACT_SWIGLU = 1, LMOE_ACT_RELU2 = 2 } lmoe_act;
typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1 } lmoe_dtype;

/* Flags of lmoe_create. */
#define LMOE_SKIP_PROJ     0x1u  /* l == d, no projections (standard MoE)       */
#define LMOE_DEBUG_CHECKS  0x2u  /* device range checks and non-finite checks   */
#define LMOE_FORCE_SIMT    0x4u  /* bf16: every contraction on the CUDA-core
                                    kernels instead of tcgen05 (for testing)    */
#define LMOE_FORCE_SWAP    0x8u  /* always use the single-CTA weight-stationary
                                    (swap-AB) expert kernels (for testing)      */
#define LMOE_FORCE_NOSWAP  0x10u /* never use the weight-stationary expert
                                    kernels (for testing)                       */
#define LMOE_FORCE_NOPAIR  0x20u /* never use the 2-SM (CTA pair) tensor-core
                                    kernels (for testing)                       */
#define LMOE_FORCE_WS_PAIR 0x40u /* expert FC1 and FC2 on the weight-stationary
                                    kernel on CTA pairs wherever the single-CTA
                                    weight-stationary kernel is not used.  It
                                    pads an expert's last tile to 16 rows, not
                                    to 128/256, but its 2-SM MMAs with N < 256
                                    run below full rate, which makes it slower
                                    at a few hundred rows per expert.           */
#define LMOE_ROUTE_FULL_SOFTMAX 0x80u  /* gates are the softmax over all N router
                                    logits taken at the k chosen experts (the
                                    paper's Eq. (1) read literally: the gates
                                    sum to less than 1) instead of the softmax
                                    renormalised over the k chosen           */
#define LMOE_ROUTE_BIAS_SELECT  0x100u /* the router bias only steers the choice
                                    (auxiliary-loss-free balancing, the
                                    paper's Section 4): experts are chosen on
                                    the fp32 sum logit + bias, the gates use
                                    the logit alone; lmoe_router_logits and
                                    the logits stage then exclude the bias,
                                    and lmoe_route_only adds the bias given to
                                    lmoe_set_weights for the choice          */
#define LMOE_EXPERTS_FP8        0x200u /* expert weights W1 and W2 as fp8 E4M3
                                    codes with one fp32 scale per output
                                    channel (lmoe_set_expert_weights_fp8);
                                    the expert MMAs run on f16 operands with
                                    fp32 accumulation.  bf16 layers with l and m multiples
                                    of 64 only (else LMOE_ERR_UNSUPPORTED)   */
#define LMOE_SINGLE_STREAM      0x400u /* every stage of lmoe_forward on the
                                    caller's stream.  By default the stages
                                    that read only x (down-projection, shared
                                    expert FC1) run on a second stream of the
                                    handle, forked from and joined back into
                                    the caller's stream inside the call, so
                                    that they overlap the router and routing
                                    steps (separate streams for the shared
                                    expert, the optimisation proposed in the
                                    paper's Section 4.3 after Table 5).
                                    Results are bitwise the same either way. */
#define LMOE_NO_PDL             0x800u /* launch the forward's kernels without
                                    programmatic dependent launch.  By
                                    default each kernel may be scheduled
                                    while its predecessor on the stream
                                    drains, sets up its barriers and tensor
                                    memory, and waits for the predecessor's
                                    writes before its first global access. */
#define LMOE_LOAD_SPLIT         0x1000u /* prefill (token-tiled) expert GEMMs
                                    split by load: the experts with more
                                    than 384 rows on CTA pairs (256-row token
                                    tiles; FC1 gathers its rows by token in
                                    both CTAs), the others on single-CTA
                                    weight-stationary tiles of their rows
                                    rounded up to 16 (at most 128 rows for a
                                    gated FC1, 256 otherwise), so an expert
                                    with few rows pays neither a 128- nor a
                                    256-row tile.  Off by default: FC1 on
                                    single-CTA 128-row tiles and FC2 on CTA
                                    pairs for every expert.  Results are the
                                    same either way up to the order of fp32
                                    sums inside the tensor cores. */
#define LMOE_NO_STREAM_K        0x2000u /* decode (weight-stationary) expert
                                    FC1 in whole tiles per CTA.  By
                                    default, with 2 to 16 tiles per CTA, the
                                    (tile, K block) units are dealt out in
                                    equal ranges, one per CTA, so the weight
                                    stream ends on every SM at the same
                                    time; a tile that straddles two ranges
                                    is summed from its two fp32 parts (in a
                                    fixed way: the result does not depend on
                                    timing).  Needs 2 x (SMs + 1) x 64 KB of
                                    workspace. */
#define LMOE_SORTED_ROWS        0x4000u /* copy the expert FC1's input rows
                                    into expert order (T*k rows of the
                                    latent width, a workspace of that size)
                                    before FC1, which then loads them as
                                    contiguous tiles by TMA instead of
                                    gathering them by token.  Off by
                                    default.  Results are the same. */
#define LMOE_EXPERTS_FP4        0x8000u /* expert weights W1 and W2 as block-
                                    scaled fp4 (MXFP4: E2M1 codes, one E8M0
                                    exponent per 32 input channels;
                                    lmoe_set_expert_weights_fp4), the format
                                    the paper's Section 2 models its experts
                                    in.  The expert MMAs run on f16 operands
                                    with fp32 accumulation, on the weight-
                                    stationary kernels at every batch size.
                                    bf16 layers with l and m multiples of
                                    512, not with LMOE_EXPERTS_FP8 or
                                    LMOE_FORCE_SIMT (else
                                    LMOE_ERR_UNSUPPORTED); no expert
                                    parallelism.                             */

#define LMOE_FC2_SPLIT          0x10000u /* prefill expert FC2 on CTA pairs:
                                    where an expert's rows past its whole
                                    256-row tiles are at most 128, they run
                                    on one 128-row single-CTA tile in a
                                    second launch (padding to 128 rows
                                    instead of 256); everything else stays
                                    on the pairs.  Results are within the
                                    bf16 tolerance of the default path. */

/* Limits of the library. */
#define LMOE_MAX_EXPERTS 1024
#define LMOE_MAX_TOPK    32

/* Bits of the device error word. */
#define LMOE_DEVERR_WAIT_TIMEOUT 0x1  /* an mbarrier wait ran past its limit     */
#define LMOE_DEVERR_RANGE        0x2  /* an index out of range (debug checks)    */
#define LMOE_DEVERR_NONFINITE    0x4  /* a NaN/Inf logit (debug checks)          */

typedef struct lmoe_layer lmoe_layer;

/*
 * lmoe_create -- a layer handle on the current CUDA device.
 * d: hidden width; l: latent width (== d with LMOE_SKIP_PROJ); N: routed
 * experts (1..LMOE_MAX_EXPERTS); k: active experts per token
 * (1..min(N, LMOE_MAX_TOPK)); m: expert width; shared_m: shared-expert width
 * (0: none).  Paper: d, l, N', K (or K'), m of Section 3; S shared experts of
 * Eq. (1) are one expert of S times the width.
 * Allocates nothing on the device.  *out receives the handle (NULL on error).
 * Errors: INVALID_ARG for any size out of range or unknown act/dtype/flag;
 * CUDA if no device is usable.
 */
lmoe_status lmoe_create(int d, int l, int N, int k, int m, lmoe_act act, int shared_m,
                        lmoe_dtype dtype, unsigned flags, lmoe_layer** out);

/*
 * lmoe_set_weights -- copy the weights into library-owned device storage
 * (repacked to the kernels' layout; the caller may free its tensors after
 * the call returns).  Synchronous: returns when the copy is done.
 *   W_g     [d, N]            router (paper W'_r, transposed)
 *   bias    [N] fp32 or NULL  additive per-expert router bias
 *   W_down  [d, l]            down-projection (NULL iff LMOE_SKIP_PROJ)
 *   W_up    [l, d]            up-projection   (NULL iff LMOE_SKIP_PROJ)
 *   W1      [N, l, m_in]      expert FC1; m_in = 2m for SwiGLU, else m
 *   W2      [N, m, l]         expert FC2
 *   Ws1     [d, ms_in]        shared FC1 (NULL iff shared_m == 0)
 *   Ws2     [shared_m, d]     shared FC2 (NULL iff shared_m == 0)
 * May be called again to replace the weights.  Allocates (once) the weight
 * storage.  Errors: INVALID_ARG (NULL where required or non-NULL where not),
 * OOM, CUDA.
 */
lmoe_status lmoe_set_weights(lmoe_layer* h, const void* W_g, const float* bias,
                             const void* W_down, const void* W_up, const void* W1,
                             const void* W2, const void* Ws1, const void* Ws2);

/*
 * lmoe_set_expert_weights_fp8 -- the expert weights of a layer created with
 * LMOE_EXPERTS_FP8 (low-precision expert weights: the paper's Section 2 models
 * FP4 expert weights, its Section 4.3 measures FP8 quantisation).  Device
 * pointers, API layout [in, out] as lmoe_set_weights:
 *   W1q [N, l, m_in] E4M3 codes (one byte each, the OCP E4M3FN encoding),
 *   W1s [N, m_in] fp32: W1[e][i][o] = value(W1q[e][i][o]) * W1s[e][o],
 *   W2q [N, m, l]    E4M3 codes,
 *   W2s [N, l] fp32: W2[e][i][o] = value(W2q[e][i][o]) * W2s[e][o].
 * The library copies (and repacks) them; the caller keeps ownership of its
 * buffers.  lmoe_set_weights is still required for the other weights (its W1
 * and W2 may then be NULL); the layer is ready once both calls succeeded.
 * Inside the expert kernels the codes widen exactly to f16 and the MMAs
 * multiply f16 operands with fp32 accumulation: the FC1 input rows are
 * converted to f16 once per forward (exact for magnitudes in [2^-14, 65504],
 * saturating above) and FC1 writes its output in f16; the scale multiplies
 * the fp32 accumulator.  Synchronous.  Errors: INVALID_ARG (NULL
 * pointer, layer created without LMOE_EXPERTS_FP8), CUDA, OOM.
 */
lmoe_status lmoe_set_expert_weights_fp8(lmoe_layer* h, const void* W1q, const float* W1s,
                                        const void* W2q, const float* W2s);

/*
 * lmoe_set_expert_weights_fp4 -- the expert weights of a layer created with
 * LMOE_EXPERTS_FP4, in the OCP microscaling format MXFP4 (the FP4 expert
 * weights the paper's Section 2 assumes for its models).  Device pointers,
 * OUTPUT-major (each weight row is one output channel, its input channels
 * contiguous), uint8:
 *   W1q [N, m_in, l / 2]  E2M1 code pairs: byte j of row o holds input
 *                         channels 2j (low nibble) and 2j + 1 (high nibble),
 *   W1e [N, m_in, l / 32] E8M0 exponents: byte b of row o scales input
 *                         channels [32 b, 32 b + 32) by 2^(byte - 127),
 *   W2q [N, l, m / 2], W2e [N, l, m / 32] the same for FC2,
 * so W1[e][i][o] = e2m1(code of channel i in row o) * 2^(W1e[e][o][i/32] - 127)
 * (E2M1: sign, 2 exponent bits, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6).  Every exponent byte must lie in [104, 140] (scales 2^-23 ..
 * 2^13, where code x scale is an f16 value; else LMOE_ERR_UNSUPPORTED).  The
 * library copies them (the caller keeps its buffers); lmoe_set_weights is
 * still required for the other weights (its W1 and W2 may be NULL).  Inside
 * the expert kernels each 32-channel block widens exactly to f16 in tensor
 * memory; the MMAs multiply f16 operands with fp32 accumulation, the FC1
 * input rows are converted to f16 once per forward and FC1 writes its output
 * in f16 (as with LMOE_EXPERTS_FP8).  Synchronous.  Errors: INVALID_ARG (NULL
 * pointer, layer created without LMOE_EXPERTS_FP4), UNSUPPORTED, CUDA, OOM.
 */
lmoe_status lmoe_set_expert_weights_fp4(lmoe_layer* h, const void* W1q, const void* W1e,
                                        const void* W2q, const void* W2e);

/*
 * lmoe_reserve -- size the workspace for up to max_T tokens per call.
 * Allocates; call it before lmoe_forward / lmoe_route_only /
 * lmoe_router_logits / lmoe_forward_host.  Calling it again with a larger
 * max_T reallocates (synchronously).  It also creates the handle's two
 * internal streams (the host entry's copy stream and the forward's side
 * stream, see LMOE_SINGLE_STREAM) and their events.  Errors: INVALID_ARG
 * (max_T < 1), OOM, CUDA.
 */
lmoe_status lmoe_reserve(lmoe_layer* h, int max_T);

/*
 * lmoe_forward -- the layer on T tokens (Eq. (1)/(2) plus the residual):
 * out[T, d] = x + MoE(x).  x and out must not alias.  0 <= T <= reserved
 * max_T (T == 0 enqueues nothing).  Errors: NOT_READY (no weights or no
 * workspace), INVALID_ARG (T out of range, NULL pointer), CUDA.
 */
lmoe_status lmoe_forward(lmoe_layer* h, const void* x, void* out, int T, lmoe_stream_t stream);

/*
 * lmoe_forward_host -- lmoe_forward with HOST buffers: copies x_host (host,
 * [T, d]) into library staging memory, runs the layer and copies the result
 * to out_host (host, [T, d]).  The upload runs on a library-owned copy stream
 * into one of two staging slots (alternating per call), so it overlaps the
 * previous call's forward; the forward and the download are enqueued on
 * stream after it.  The caller synchronises stream before reading out_host or
 * reusing x_host.  Pinned host memory makes the copies asynchronous.  Calls
 * on one handle must come from one host thread at a time.  Errors: as
 * lmoe_forward.
 */
lmoe_status lmoe_forward_host(lmoe_layer* h, const void* x_host, void* out_host, int T,
                              lmoe_stream_t stream);

/*
 * lmoe_route_only -- the routing steps on given fp32 logits [T, N]
 * (Section 3: the top-K set and the dispatch grouping):
 *   idx[T, k]     experts of each token in slot order (logit desc, index asc;
 *                 +0.0 == -0.0)
 *   w[T, k]       renormalised gates exp(l_j - l_0) / sum_j' exp(l_j' - l_0)
 *   offsets[N+1]  first expert-sorted row of each expert; offsets[N] = T*k
 *   perm[T*k]     expert-sorted row -> pair t*k + j; within one expert rows
 *                 are in ascending token order
 * The same kernels lmoe_forward routes with.  Logits must be finite (with
 * LMOE_DEBUG_CHECKS a non-finite logit sets LMOE_DEVERR_NONFINITE).
 * Errors: NOT_READY (no workspace), INVALID_ARG.
 */
lmoe_status lmoe_route_only(lmoe_layer* h, const float* logits, int T, int* idx, float* w,
                            int* offsets, int* perm, lmoe_stream_t stream);

/*
 * lmoe_router_logits -- the router GEMM alone: logits[T, N] (fp32) =
 * x Wg + bias, computed by the kernel lmoe_forward uses (deterministic run to
 * run).  Errors: NOT_READY, INVALID_ARG.
 */
lmoe_status lmoe_router_logits(lmoe_layer* h, const void* x, float* logits, int T,
                               lmoe_stream_t stream);

/* Intermediate buffers of the last lmoe_forward, for tests and debugging. */
typedef enum {
  LMOE_STAGE_LOGITS = 0,   /* [T, N]   fp32                                  */
  LMOE_STAGE_IDX = 1,      /* [T, k]   int32                                 */
  LMOE_STAGE_W = 2,        /* [T, k]   fp32                                  */
  LMOE_STAGE_OFFSETS = 3,  /* [N+1]    int32                                 */
  LMOE_STAGE_PERM = 4,     /* [T*k]    int32 sorted row -> t*k+j             */
  LMOE_STAGE_Z = 5,        /* [T, l]   dtype  latent rows (not with SKIP)    */
  LMOE_STAGE_H = 6,        /* [T*k, m] dtype  expert hidden rows, sorted
                              (f16 with LMOE_EXPERTS_FP8 / _FP4)            */
  LMOE_STAGE_YS = 7,       /* [T*k, l] dtype  gate-scaled expert outputs,
                                             expert-sorted rows (as H)       */
  LMOE_STAGE_COMB = 8      /* [T, l]   dtype  combined rows (not with SKIP)  */
} lmoe_stage;

/*
 * lmoe_stage_bytes -- size in bytes of a stage buffer for T tokens.
 * lmoe_debug_dump -- copy that buffer of the last forward (T of that call)
 * into dst (device, at least lmoe_stage_bytes bytes), on stream.
 * Errors: INVALID_ARG (unknown or absent stage, bytes too small), NOT_READY.
 */
lmoe_status lmoe_stage_bytes(const lmoe_layer* h, int stage, int T, size_t* bytes);
lmoe_status lmoe_debug_dump(lmoe_layer* h, int stage, void* dst, size_t bytes,
                            lmoe_stream_t stream);

/*
 * lmoe_last_error -- synchronise the device, read the device error word into
 * *device_error_word (LMOE_DEVERR_* bits, 0 when clean) and clear it.
 * Returns TIMEOUT or DEVICE when a bit was set, CUDA if the device itself
 * reports an error, OK otherwise.
 */
lmoe_status lmoe_last_error(lmoe_layer* h, int* device_error_word);

/*
 * Per-stage timing.  lmoe_profile_begin allocates CUDA events for up to
 * max_forwards calls (synchronous); afterwards every lmoe_forward records an
 * event at each stage boundary on its stream.  lmoe_profile_end synchronises,
 * writes the stage durations in milliseconds to ms[f * n_stages + s] for the
 * recorded forwards f (at most capacity values), sets *n_forwards and
 * *n_stages, and stops recording.  Stage s is named by lmoe_stage_name(s).
 */
lmoe_status lmoe_profile_begin(lmoe_layer* h, int max_forwards);
/*
 * lmoe_profile_begin_stages -- lmoe_profile_begin recording only the
 * boundaries of the stages whose bit is set in stage_mask (bit s = stage s);
 * lmoe_profile_end writes -1 for the other stages.  An event recorded between
 * two kernels makes the second wait for the first to finish, so timing one
 * stage this way leaves the other kernel boundaries free to launch early.
 * Errors: INVALID_ARG (max_forwards < 1, stage_mask without a stage bit).
 */
lmoe_status lmoe_profile_begin_stages(lmoe_layer* h, int max_forwards, unsigned stage_mask);
lmoe_status lmoe_profile_end(lmoe_layer* h, float* ms, int capacity, int* n_forwards,
                             int* n_stages);
const char* lmoe_stage_name(int stage);

/*
 * ---- Expert parallelism: dispatch and combine in latent space ----
 *
 * The paper's deployment analysis (LatentMoE, Section 2.2 "Communication
 * Bottleneck"; Section 3, the paragraph after Eq. (1)) splits the N experts
 * over `world` GPUs and moves, per token, its routed rows to the GPUs that
 * own its experts and the expert outputs back; LatentMoE does both in the
 * latent width l instead of d, so both all-to-alls carry d / l times fewer
 * bytes.  These calls run one rank's compute; the caller moves the rows
 * between ranks (an all-to-all: NCCL through torch.distributed, see
 * mixture_experts_layer_64_b200/ep.py).  Rows a rank receives must be in
 * its own device memory before lmoe_ep_experts reads them.
 *
 * Ownership: N % world == 0 and rank r owns the n = N / world experts
 * [r n, (r + 1) n).  Every rank's handle holds the weights of all N experts
 * (lmoe_set_weights); lmoe_ep_experts reads those of its own n only.
 * Per call, on every rank:
 *   1 lmoe_ep_dispatch: router, top-k, grouping, down-projection (and the
 *     shared expert's first matrix).  send_rows[r] = the latent row of the
 *     token of sorted row r (rows sorted by expert, then token; with
 *     LMOE_SKIP_PROJ the token's row of x), send_gates[r] = its gate,
 *     expert_counts[e] = the rows routed to expert e.  The rows for rank q are
 *     the contiguous block of its experts.
 *   2 (caller) every rank sends rank q the n counts of q's experts: rank q
 *     holds recv_counts[s][e] (s = source rank); then the row blocks and
 *     gates, sources in rank order.
 *   3 lmoe_ep_experts: the n local experts' FFNs on the received rows, with
 *     each row's gate applied; out_rows[i] belongs to received row i.
 *   4 (caller) the reverse exchange: each source receives back its rows in
 *     the order it sent them (its send_rows order).
 *   5 lmoe_ep_combine: per token the sum of its k returned rows, the
 *     up-projection, the shared expert and the residual.
 * Steps 1 and 5 pair up on one handle (5 uses 1's routing); one dispatch at
 * a time per handle.  All pointers are device pointers, rows in the layer
 * dtype with row stride l (d with LMOE_SKIP_PROJ), counts int32.
 */

/* Sizes the expert-side workspace for up to max_recv_rows received rows per
 * call (at most world * T * k).  Allocates.  Errors: INVALID_ARG, NOT_READY
 * (call lmoe_reserve first), OOM, CUDA. */
lmoe_status lmoe_ep_reserve(lmoe_layer* h, int max_recv_rows);

/* Step 1.  send_rows [T*k, l], send_gates [T*k] fp32, expert_counts [N]
 * int32: device outputs owned by the caller.  0 < T <= reserved max_T.
 * Errors: NOT_READY, INVALID_ARG, UNSUPPORTED (fp8 expert weights), CUDA. */
lmoe_status lmoe_ep_dispatch(lmoe_layer* h, const void* x, int T, void* send_rows,
                             float* send_gates, int* expert_counts, lmoe_stream_t stream);

/* Step 3.  recv_counts: HOST array [world, n] int32, recv_counts[s][e] =
 * the rows source rank s sent for local expert e (the caller has them: they
 * size the all-to-all); Rr = their sum <= the reserved max_recv_rows.
 * recv_rows [Rr, l] and recv_gates [Rr] (device) in received order: sources
 * in rank order, each source's rows as it sent them.  out_rows [Rr, l]
 * (device): the gate-scaled expert outputs in received order.  The local
 * experts' kernels are chosen from the mean received rows per local expert
 * as in lmoe_forward.  The small grouping tables are uploaded from a
 * library-owned pinned buffer (the call waits for the previous call's upload
 * before rewriting it).  Errors: NOT_READY (no lmoe_ep_reserve),
 * INVALID_ARG (sizes, NULL, negative counts, N % world != 0),
 * UNSUPPORTED (Rr over the reserved size; fp8 expert weights), CUDA. */
lmoe_status lmoe_ep_experts(lmoe_layer* h, const void* recv_rows, const float* recv_gates,
                            const int* recv_counts, int rank, int world, void* out_rows,
                            lmoe_stream_t stream);

/* Step 5.  back_rows [T*k, l] in the dispatch's send order; x the same
 * [T, d] input as the dispatch, out [T, d].  Errors: NOT_READY (no matching
 * dispatch), INVALID_ARG, CUDA. */
lmoe_status lmoe_ep_combine(lmoe_layer* h, const void* x, const void* back_rows, void* out, int T,
                            lmoe_stream_t stream);

/* Host-side plan of step 3 (no GPU, host pointers): the order in which the
 * received rows are grouped by local expert -- experts in order, then
 * sources in rank order, each source's rows as sent.  recv_counts [world,
 * n]; offsets [n + 1] (offsets[n] = Rr); perm [Rr]: grouped row -> received
 * row.  lmoe_ep_experts builds the same order on the device.  Errors:
 * INVALID_ARG (bad sizes, NULL, negative counts). */
lmoe_status lmoe_ep_local_plan(const int* recv_counts, int world, int n_local, int* offsets,
                               int* perm);

/*
 * lmoe_route_only_noalloc -- lmoe_route_only without a handle and without
 * allocating device memory.  The paper has no counterpart: this is an
 * interface for callers, not a step of the method.
 *
 * Some callers cannot call cudaMalloc: an inference server that reserves all
 * of HBM for its own pool up front (a driver allocation would fail or
 * fragment it), or code running where the device-wide synchronisation that
 * cudaMalloc / cudaFree imply is not allowed.  This call runs the routing
 * kernels of lmoe_route_only (same arguments and results: idx, w, offsets,
 * perm for N experts and top-k) with their scratch in a fixed file-scope
 * device array of LMOE_NOALLOC_SCRATCH_BYTES, which every GPU that loads the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   Limits: N <= LMOE_MAX_EXPERTS, k <= LMOE_MAX_TOPK and
 *   N * ceil(T / 32) <= LMOE_NOALLOC_MAX_WORDS (e.g. T <= 8192 with N = 1024,
 *   T <= 16384 with N = 512); beyond them it returns LMOE_ERR_UNSUPPORTED and
 *   enqueues nothing.
 *   Setup: every call looks up the array's device address
 *   (cudaGetSymbolAddress) on the current device, so it stays valid across a
 *   device reset; the first call on a device also loads the module there:
 *   make that first call before any stream capture.  The current device
 *   must be the one that holds the pointers and the stream.
 *   Sharing: every call uses the same array and clears the parts that must
 *   start at zero, so calls that overlap on the GPU (other streams, other
 *   host threads) race and must be serialised by the caller.
 * error_word: a caller-owned device int, or NULL.  When given, the call
 * zeroes it on the stream and runs the kernels with the device checks of
 * LMOE_DEBUG_CHECKS: a non-finite logit sets LMOE_DEVERR_NONFINITE and an
 * expert index out of range LMOE_DEVERR_RANGE in it.  The call itself does
 * not synchronise: read the word once the stream has completed.  With NULL
 * no checks run, and non-finite logits give indices that are in range but
 * otherwise unspecified.
 * Errors: INVALID_ARG (bad sizes, NULL pointers), UNSUPPORTED (over the
 * limits), CUDA (a failed enqueue: the outputs are then not written).
 */
#define LMOE_NOALLOC_MAX_WORDS     262144u
#define LMOE_NOALLOC_SCRATCH_BYTES 3211264u
lmoe_status lmoe_route_only_noalloc(const float* logits, int T, int N, int k, int* idx, float* w,
                                    int* offsets, int* perm, int* error_word,
                                    lmoe_stream_t stream);

/*
 * lmoe_selftest_wait_timeout -- test hook for the bounded waits: enqueues one
 * kernel whose thread waits on an mbarrier that nothing arrives on; after
 * limit_us microseconds (1 .. 1e6) the wait gives up, sets
 * LMOE_DEVERR_WAIT_TIMEOUT in the handle's device error word and the kernel
 * returns, leaving the context usable.  lmoe_last_error then returns
 * LMOE_ERR_TIMEOUT.  No counterpart in the paper (a property of this
 * implementation: no wait in the library's kernels can hang a GPU).
 * Errors: INVALID_ARG (limit out of range), NOT_READY (no workspace), CUDA.
 */
lmoe_status lmoe_selftest_wait_timeout(lmoe_layer* h, unsigned limit_us, lmoe_stream_t stream);

/* Kernel launches the last lmoe_forward enqueued (library kernels only). */
int lmoe_last_launch_count(const lmoe_layer* h);

/* Which expert kernels the last lmoe_forward used, FC1 in bits 0-2 and FC2
 * in bits 3-5, each: 0 CUDA-core, 1 tcgen05 token-tiled, 2 tcgen05
 * weight-stationary (swap-AB), 3 tcgen05 token-tiled on CTA pairs (2-SM MMA),
 * 4 tcgen05 weight-stationary on CTA pairs (the expert's rows as the MMA's N,
 * split into tiles of nearly equal size in units of 16 rows), 5 tcgen05
 * split by load (CTA-pair token tiles for the experts with more than 384
 * rows, single-CTA weight-stationary tiles of up to 128 / 256 rows for the
 * others). */
int lmoe_last_expert_path(const lmoe_layer* h);

const char* lmoe_status_string(lmoe_status s);

/* Text of the last host-side failure on h (the failing CUDA call and its
 * message); "" when none.  Valid until the next call on h. */
const char* lmoe_error_detail(const lmoe_layer* h);

/* Frees everything the handle owns (synchronises its device). NULL is a no-op. */
void lmoe_destroy(lmoe_layer* h);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H */
