/*
 * moe.h - C ABI of the B200 (sm_100a) DeepSeek-V3 MoE layer forward pass.
 *
 * The layer, as the pages define it:
 *   - "DeepSeek-V3" (ainfra.dev llm-vis): "Mixture-of-Experts FFN" box (forward:
 *     router, routed experts, shared expert), "MoE router" box (sigmoid scores,
 *     selection-only bias, renormalised weights, routed scaling x2.5, router in
 *     fp32), "Routed experts" box (grouped dispatch of all tokens per expert),
 *     "Shared expert" box, "Expert combine" box
 *     (y = 2.5 * sum_i w_i e_i(x) + shared(x)), "SwiGLU MLP" box
 *     (W_down(SiLU(W_gate x) * W_up x)), "Residual add" box.
 *   - "DeepSeek V3" field guide (curiouscaliboi), cutaway 02 "Fine-grained expert
 *     routing": 8 groups of 32, each scored by its two strongest bias-adjusted
 *     expert scores, top 4 groups eligible, top 8 experts inside them, weights
 *     from the unbiased sigmoid renormalised to one, no token dropped.
 *   - "Teardown: DeepSeek-V3", section 6 (sizes, bias for selection only) and
 *     section 10 (FP8: E4M3, 1x128 activation tiles, 128x128 weight blocks,
 *     router in higher precision).
 *
 * Conventions shared by every entry point
 *   - All array arguments are DEVICE pointers (cudaMalloc'd or torch tensors'
 *     data_ptr), row-major and densely packed, owned by the caller.  The
 *     library allocates no device memory per call and keeps no per-call state.
 *     Tensor-operand pointers (x, weights, workspace) must be 16-byte aligned.
 *   - Every call is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns without synchronising the host.
 *   - Errors found on the host (bad sizes, NULL or misaligned pointers) return
 *     MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED before anything is enqueued.
 *     A failed launch returns MOE_ERR_CUDA.  Errors found on the device (an
 *     expert id out of range, a pipeline wait that ran past its time limit) set
 *     bits in a per-device error word that moe_device_error() reads; kernels
 *     never trap.
 *   - T = 0 is valid and enqueues nothing.
 *   - Requires an sm_100 device (B200); other devices get MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t;   /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* NULL / misaligned pointer, inconsistent sizes */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype combination, device) */
    MOE_ERR_WORKSPACE = 3,     /* workspace smaller than moe_workspace_size() */
    MOE_ERR_DEVICE = 4,        /* the device error word is non-zero */
    MOE_ERR_CUDA = 5           /* a CUDA runtime call or launch failed */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2 } moe_dtype;

/* Device error word bits (moe_device_error). */
#define MOE_DEVERR_BAD_EXPERT 0x1u    /* a routed expert id outside [0, n_experts) */
#define MOE_DEVERR_TIMEOUT    0x2u    /* a pipeline wait exceeded its limit */
#define MOE_DEVERR_BAD_ROWS   0x4u    /* a schedule entry or a combine row's token outside its buffer */
#define MOE_DEVERR_NONFINITE  0x8u    /* a router logit was NaN or infinite (a NaN ranks last) */
#define MOE_DEVERR_BOUNDS     0x10u   /* checking build only: a table entry, row range or TMA
                                         coordinate outside its buffer (the access was skipped
                                         or replaced by an in-bounds one) */

/* Layer shape ("Teardown: DeepSeek-V3", At a glance + section 6; field guide
 * cutaway 02).  Constraints checked by every entry point:
 *   d % 128 == 0, hidden % 128 == 0, shared_hidden % 128 == 0 (0 if n_shared = 0),
 *   n_experts <= 1024, n_experts % n_groups == 0, group size >= 2, n_groups <= 32,
 *   1 <= topk_groups <= n_groups, 1 <= top_k <= min(32, topk_groups * group size),
 *   n_shared in {0, 1}, act_dtype in {F32, BF16}, weight_dtype in {BF16, E4M3}. */
typedef struct {
    int d;               /* model width (7168) */
    int n_experts;       /* routed experts E (256) */
    int n_groups;        /* expert groups G (8) */
    int topk_groups;     /* eligible groups per token (4) */
    int top_k;           /* routed experts per token k (8) */
    int hidden;          /* routed expert SwiGLU width H (2048) */
    int n_shared;        /* shared experts, 0 or 1 (1) */
    int shared_hidden;   /* shared expert width Hs (2048) */
    float routed_scale;  /* routed scaling factor (2.5) */
    moe_dtype act_dtype;     /* x: MOE_F32 or MOE_BF16 */
    moe_dtype weight_dtype;  /* routed + shared expert weights: MOE_BF16 or MOE_E4M3 */
} moe_config;

/* Layer weights, nn.Linear layout ([out, in], K contiguous), experts stacked.
 * The router weight is always bf16 (the router stays in high precision).
 * E4M3 expert weights come with one fp32 scale per 128x128 block. */
typedef struct {
    const void* w_router;   /* [E, d] bf16 */
    const void* w_gate;     /* [E, H, d] bf16 | e4m3 */
    const void* w_up;       /* [E, H, d] bf16 | e4m3 */
    const void* w_down;     /* [E, d, H] bf16 | e4m3 */
    const float* s_gate;    /* e4m3 only: [E, H/128, d/128] */
    const float* s_up;      /* e4m3 only: [E, H/128, d/128] */
    const float* s_down;    /* e4m3 only: [E, d/128, H/128] */
    const void* ws_gate;    /* shared expert [Hs, d] */
    const void* ws_up;      /* shared expert [Hs, d] */
    const void* ws_down;    /* shared expert [d, Hs] */
    const float* ss_gate;   /* e4m3 only: [Hs/128, d/128] */
    const float* ss_up;     /* e4m3 only: [Hs/128, d/128] */
    const float* ss_down;   /* e4m3 only: [d/128, Hs/128] */
} moe_weights;

/* Bytes of device workspace moe_forward needs for up to T_max tokens
 * (0 on invalid config).  The workspace holds the router logits, the routing,
 * the permutation, the tile schedule, the permuted activations, the SwiGLU
 * output h and the fp32 combine buffer. */
MOE_API size_t moe_workspace_size(const moe_config* cfg, int T_max);

/* Stages 1+2: router and selection ("MoE router" box; field guide cutaway 02).
 *   x != NULL: logits[T,E] (fp32, written) = x[T,d] . w_router[E,d]^T with fp32
 *              accumulation; x is cfg->act_dtype (fp32 or bf16).
 *   x == NULL: logits[T,E] is an input (logits-in mode).
 * Then s = sigmoid(logits); b = s + bias (selection only); group score = sum of
 * the two largest b in the group; the topk_groups best groups are eligible;
 * topk_idx[T,k] (int32) = the k best experts by b among them, in descending b
 * (ties: lower index first); topk_w[T,k] (fp32) = s[idx] / sum of the selected
 * s taken in ascending expert index, so the weights sum to 1 and are NOT
 * multiplied by routed_scale.  The sigmoid is a fixed fp32 formula (Cody-Waite
 * reduction and a degree-7 Taylor polynomial, correctly rounded operations
 * only), so identical logits give bit-identical idx and w on any device.
 * bias: [E] fp32.  Logits must be finite. */
MOE_API moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router, float* logits,
                     const float* bias, int T, int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Stage 3: permutation ("Routed experts" box: group all tokens per expert).
 * Counting sort of the T*k (token, slot) pairs by expert, ascending token
 * inside each expert (the order is unique: a token picks an expert once).
 *   counts[E]    number of pairs per expert
 *   offsets[E+1] exclusive prefix sum of counts; offsets[E] = T*k
 *   src[T*k]     src[row] = t*k + j for the pair in permuted position row
 *   inv[T*k]     inv[t*k + j] = row
 * An id outside [0, E) sets MOE_DEVERR_BAD_EXPERT and is skipped. */
MOE_API moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int T, int32_t* counts,
                       int32_t* offsets, int32_t* src, int32_t* inv, moe_stream_t stream);

/* Stages 1-5: the whole layer ("Mixture-of-Experts FFN" forward; "Expert
 * combine" box; "Residual add" box):
 *   y[t] (+)= routed_scale * sum_j w[t,j] * expert_{idx[t,j]}(x[t]) + shared(x[t])
 * expert(x) = W_down (SiLU(W_gate x) * (W_up x)), SiLU(z) = z * sigmoid(z).
 * x: [T, d] cfg->act_dtype (fp32 input is rounded to bf16 for the experts; with
 * E4M3 weights x must be bf16 and is quantised to e4m3 per token and
 * 128-channel block as moe_quantize_act does, the expert GEMMs run on e4m3
 * tensor cores with the partial sums of every 128-element K block promoted
 * to fp32 with both block scales, and h is stored as e4m3 with one scale per
 * row and 128 features).
 * y: [T, d] in y_dtype (MOE_F32 or MOE_BF16); accumulate = 0 overwrites y,
 * accumulate = 1 adds the layer output to y (the residual stream).
 * The expert GEMMs run on tcgen05 tensor cores with fp32 accumulation; h is
 * stored in bf16 (e4m3 with 1x128 scales for E4M3 weights).  The combine adds
 * fp32 partial sums with atomics, so the summation order of a token's 9
 * expert outputs may vary between runs (within fp32 rounding).
 * workspace: device buffer of ws_bytes >= moe_workspace_size(cfg, T),
 * 256-byte aligned; it is overwritten. */
MOE_API moe_status moe_forward(const moe_config* cfg, const moe_weights* w, const void* x, const float* bias,
                       int T, void* y, moe_dtype y_dtype, int accumulate, void* workspace,
                       size_t ws_bytes, moe_stream_t stream);

/* Stage 6, FP8 layers ("Teardown: DeepSeek-V3", section 10: activations in
 * E4M3 scaled per 1x128 tile).  For every token t and 128-channel block b of
 * x [T, d] bf16 (d % 128 == 0):
 *   sx[t, b] = amax_b / 448 (1 when the block is all zero)   fp32 [T, d/128]
 *   q[t, c]  = e4m3_rn_sat(x[t, c] / sx[t, b])               uint8 [T, d]
 * The divides are correctly rounded fp32 and the conversion rounds to nearest
 * even with saturation at +-448 (OCP E4M3), so the codes are reproducible bit
 * for bit.  moe_forward with E4M3 weights runs the same kernel. */
MOE_API moe_status moe_quantize_act(const void* x, int T, int d, uint8_t* q, float* sx, moe_stream_t stream);

/* Bias controller ("DeepSeek-V3" llm-vis, "MoE router" box, update_bias;
 * "Teardown: DeepSeek-V3", section 6: after each step the selection bias is
 * lowered for overloaded experts and raised for underloaded ones).  With the
 * per-expert token counts of a batch (moe_permute's counts, or the forward's
 * via moe_routing_out):
 *   mean = (sum of counts) / E                  (fp32)
 *   bias[e] = counts[e] > mean ? bias[e] - gamma : bias[e] + gamma   (fp32)
 * counts: [E] int32; bias: [E] fp32, updated in place; gamma: the step (the
 * pages use 1e-3).  Deterministic: same inputs, same bits. */
MOE_API moe_status moe_update_bias(const moe_config* cfg, const int32_t* counts, float* bias, float gamma,
                                   moe_stream_t stream);

/* The kernels moe_forward runs for T tokens on the current device: which
 * grouped-GEMM variant, its token tile, the router's K splits, the
 * permutation's CTA count and how many kernels one call launches.  A pure
 * host-side query (no launch, no allocation); T == 0 gives all zeros. */
typedef struct moe_plan {
    int token_tile;    /* token rows per grouped-GEMM tile (BN: 32, 64, 128 or 256) */
    int cta_pair;      /* 1: the grouped GEMMs run on CTA pairs (tcgen05 cta_group::2) */
    int fp8;           /* 1: e4m3 expert GEMMs with block scales */
    int router_splits; /* K splits of the router GEMM, reduced in a fixed order (1: none) */
    int permute_ctas;  /* CTAs of the permutation (1: the single-CTA kernel) */
    int launches;      /* kernels one moe_forward call launches */
} moe_plan;
MOE_API moe_status moe_forward_plan(const moe_config* cfg, int T, moe_dtype y_dtype, moe_plan* plan);

/* Self-test of the failure path every in-kernel wait has: one kernel waits on
 * an mbarrier that nothing completes, gives up after limit_ns (at most 1 s)
 * and sets MOE_DEVERR_TIMEOUT in the device error word (read it with
 * moe_device_error); the context stays usable.  Nothing else runs in it. */
MOE_API moe_status moe_selftest_wait_timeout(unsigned long long limit_ns, moe_stream_t stream);

/* Number of kernels this library has launched in this process, over all
 * devices and streams (a diagnostic counter; never reset). */
MOE_API unsigned long long moe_launch_count(void);

/* Stage timing for moe_forward_ex: six CUDA events (cudaEvent_t handles,
 * created by the caller) that the call records on `stream`:
 *   ev[0] before the router          ev[3] after the gate/up GEMM (SwiGLU)
 *   ev[1] after the selection        ev[4] after the down GEMM and combine
 *   ev[2] after permutation + gather ev[5] after the output cast
 * so that cudaEventElapsedTime(ev[i], ev[i+1]) is the device time of a stage. */
typedef struct CUevent_st* moe_event_t;
typedef struct {
    moe_event_t ev[6];
} moe_stage_events;

/* Optional outputs of moe_forward_ex: the routing and permutation the layer
 * used.  Each non-NULL pointer is a caller device buffer that receives, exactly
 * as the layer computed and consumed them: the router logits [T, E] fp32,
 * topk_idx [T, k] int32, topk_w [T, k] fp32 (unscaled), and the permutation
 * counts [E], offsets [E+1], src [T*k], inv [T*k] int32 as moe_permute defines
 * them.  (moe_route runs the router without splitting K, so its logits may
 * differ from these in the last bits.) */
typedef struct {
    float* logits;
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* src;
    int32_t* inv;
} moe_routing_out;

/* moe_forward, recording the stage events when `events` is not NULL and
 * writing its routing into `routing` when that is not NULL. */
MOE_API moe_status moe_forward_ex(const moe_config* cfg, const moe_weights* w, const void* x, const float* bias,
                                  int T, void* y, moe_dtype y_dtype, int accumulate, void* workspace,
                                  size_t ws_bytes, moe_stream_t stream, const moe_stage_events* events,
                                  const moe_routing_out* routing);

/* Bytes of device workspace moe_forward_host needs for up to T_max tokens with
 * output type y_dtype: moe_workspace_size(cfg, T_max) plus the device copies of
 * x and y, each rounded up to 256 bytes (0 on invalid arguments). */
MOE_API size_t moe_host_workspace_size(const moe_config* cfg, int T_max, moe_dtype y_dtype);

/* moe_forward on host buffers: the layer as a host program calls it, with the
 * activations in host memory and the weights, the bias and the workspace on
 * the device.  This entry point has no counterpart on the pages; it is the
 * copy in, the layer of moe_forward and the copy out in one call.
 *   x_host [T, d] cfg->act_dtype and y_host [T, d] y_dtype are host memory.
 *   The call enqueues on `stream`: the copy of x_host into the workspace, with
 *   accumulate = 1 the copy of y_host in (the residual), moe_forward on the
 *   device copies, and the copy of the result back into y_host.  It returns
 *   without waiting: y_host holds the result once the stream has passed that
 *   work (cudaStreamSynchronize, or an event recorded after the call), and
 *   both host buffers must stay valid and untouched until then.
 *   With page-locked host memory (cudaHostAlloc, cudaHostRegister) the copies
 *   run on the copy engines while other streams compute, so two calls on two
 *   streams with two workspaces overlap one call's copies with the other's
 *   kernels.  With pageable memory the driver stages the copies and the call
 *   may block the host until they are done.
 *   workspace: device, 256-byte aligned, ws_bytes >= moe_host_workspace_size(
 *   cfg, T, y_dtype); its tail holds the device copies of x and y.
 * Every argument is checked before anything is enqueued; results and errors as
 * moe_forward, MOE_ERR_CUDA when a copy cannot be enqueued. */
MOE_API moe_status moe_forward_host(const moe_config* cfg, const moe_weights* w, const void* x_host,
                                    const float* bias, int T, void* y_host, moe_dtype y_dtype, int accumulate,
                                    void* workspace, size_t ws_bytes, moe_stream_t stream);

/* Pre-norm ("DeepSeek-V3" llm-vis, "RMSNorm" box: every token vector is
 * rescaled to unit RMS over its features with eps = 1e-6, cast back to bf16,
 * then multiplied by the learned per-feature gain):
 *   r_t      = 1 / sqrt(mean_c h[t,c]^2 + eps)      (fp32 reduction, correctly
 *                                                    rounded divide and rsqrt)
 *   out[t,c] = bf16( bf16(h[t,c] * r_t) * g[c] )
 * h, out: [T, d] bf16 row-major (must not overlap); g: [d] bf16; all 16-byte
 * aligned; d a multiple of 8 and at most 8192.  With q and sx (both or
 * neither; d a multiple of 128) the same pass also writes the 1x128 e4m3 codes
 * and scales of `out`, bit for bit as moe_quantize_act(out) would. */
MOE_API moe_status moe_rmsnorm(const void* h, const void* g, float eps, int T, int d, void* out, uint8_t* q,
                               float* sx, moe_stream_t stream);

/* The MoE sublayer of a pre-norm decoder block ("Residual add" box: the
 * sublayer reads norm2(h) and its output is added to the untouched stream h):
 *   y = bf16( h + MoE(RMSNorm(h; norm_g, eps)) )
 * with MoE as moe_forward computes it (routing, experts, combine) on the
 * normalised activations; in the FP8 layer the norm also produces the e4m3
 * activations (one pass).  h: [T, d] bf16 (cfg->act_dtype must be MOE_BF16);
 * norm_g: [d] bf16; y: [T, d] bf16 and may be h itself (the residual stream
 * updated in place).  workspace: moe_block_workspace_size(cfg, T) bytes,
 * 256-byte aligned.  events / routing as in moe_forward_ex (the norm runs in
 * the first stage). */
MOE_API size_t moe_block_workspace_size(const moe_config* cfg, int T_max);
MOE_API moe_status moe_forward_block(const moe_config* cfg, const moe_weights* w, const void* norm_g, float eps,
                                     const void* h, const float* bias, int T, void* y, void* workspace,
                                     size_t ws_bytes, moe_stream_t stream, const moe_stage_events* events,
                                     const moe_routing_out* routing);

/* Dense SwiGLU FFN ("DeepSeek-V3" llm-vis, "SwiGLU MLP" box; the model's first
 * layers use a dense FFN of hidden width 18432 in place of the experts):
 *   y (+)= W_down ( SiLU(W_gate x) * (W_up x) )
 * on the same grouped-GEMM kernels as the experts (one group of all T rows).
 * w_gate, w_up: [hidden, d]; w_down: [d, hidden] (nn.Linear layout), bf16, or
 * e4m3 codes with s_gate, s_up [hidden/128, d/128] and s_down [d/128, hidden/128]
 * fp32 block scales (weight_dtype MOE_E4M3; x is then quantised per 1x128 tile
 * and h stored as e4m3 with 1x128 scales, as in the FP8 layer).  x: [T, d]
 * (MOE_BF16, or MOE_F32 rounded to bf16; FP8 needs bf16); y: [T, d] fp32 or
 * bf16, `accumulate` adds into it.  d and hidden multiples of 128.  h is
 * stored in bf16 between the projections.  workspace: moe_dense_workspace_size
 * bytes, 256-byte aligned.  events (optional) as in moe_forward_ex: ev[0] = ev[1]
 * (no router), ev[2] after the table setup and the gather.  Errors as
 * moe_forward. */
MOE_API size_t moe_dense_workspace_size(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype, int T_max);
MOE_API moe_status moe_dense_ffn(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype, const void* w_gate,
                                 const void* w_up, const void* w_down, const float* s_gate, const float* s_up,
                                 const float* s_down, const void* x, int T, void* y, moe_dtype y_dtype,
                                 int accumulate, void* workspace, size_t ws_bytes, moe_stream_t stream,
                                 const moe_stage_events* events);

/* ---------------------------------------------------------------- expert parallelism
 * The routed experts split over n_ranks ranks (one process per GPU) in
 * contiguous blocks of E / n_ranks.  With n_ranks = n_groups rank r holds group
 * r: the pages' groups are device-aligned ("DeepSeek-V3" llm-vis, "MoE router"
 * box), so a token reaches at most topk_groups ranks.  One layer forward on a
 * rank: moe_route on its own tokens -> moe_ep_dispatch -> all-to-all of the
 * counts and the rows (the caller's collective, e.g. NCCL) -> moe_experts_routed
 * on the received rows -> all-to-all of the results back -> the shared expert
 * on the rank's own tokens (moe_dense_ffn into an fp32 y_acc) -> moe_ep_combine.
 * The result equals moe_forward's up to the order of the fp32 additions. */

/* Most send rows moe_ep_dispatch produces for T tokens: T * min(k, n_ranks)
 * (0 on invalid arguments). */
MOE_API int moe_ep_max_send_rows(const moe_config* cfg, int T, int n_ranks);

/* Dispatch.  For each rank q = 0 .. n_ranks-1, the tokens with at least one of
 * their k selected experts in q's block [q E/n_ranks, (q+1) E/n_ranks), each
 * once, in ascending token order; the rows are rank-major:
 *   topk_idx [T, k] int32, topk_w [T, k] fp32  moe_route's routing (ids outside
 *                                              [0, E) are ignored)
 *   x [T, d] cfg->act_dtype                    the rank's activations
 *   send_counts [n_ranks], send_offsets [n_ranks + 1] (exclusive prefix sum;
 *                                              send_offsets[n_ranks] = rows)
 *   send_tok [rows]    origin token of each row
 *   send_x [rows, d]   bf16 rows of x (fp32 x rounded to bf16, as the experts round it)
 *   send_idx [rows, k], send_w [rows, k]  the token's whole routing (the
 *                                         receiver keeps the slots of its block)
 * The row arrays hold moe_ep_max_send_rows rows; counts and offsets are written
 * for T = 0 too.  n_ranks in [1, 32] and dividing E; x and send_x 16-byte aligned. */
MOE_API moe_status moe_ep_dispatch(const moe_config* cfg, int n_ranks, const int32_t* topk_idx, const float* topk_w,
                                   const void* x, int T, int32_t* send_counts, int32_t* send_offsets,
                                   int32_t* send_tok, void* send_x, int32_t* send_idx, float* send_w,
                                   moe_stream_t stream);

/* Fixed-capacity, packed dispatch: the same rows as moe_ep_dispatch, laid out so
 * that the exchange needs no row counts on the host (equal-sized all-to-all
 * blocks, capturable in a CUDA graph).  Rank q's rows occupy slots
 * [q * capacity, q * capacity + send_counts[q]) in ascending token order; the
 * other slots of its block are padding.  Each slot is one packed row of
 * moe_ep_packed_row_bytes(cfg) bytes:
 *   bf16 x [d] (fp32 x rounded to bf16) | int32 expert ids [k] | fp32 weights [k] | padding to 16 B
 * a padding slot has send_tok = -1 and all k ids -1 (its x and weights are
 * unspecified), so a receiver skips it without knowing the counts.
 *   send_counts [n_ranks]       rows for each rank (for the caller's bookkeeping)
 *   send_tok [n_ranks*capacity] origin token of each slot, -1 for padding
 *   packed [n_ranks*capacity, row_bytes], 16-byte aligned
 * capacity >= T (a token goes to a rank at most once) and the same on every
 * rank.  Errors as moe_ep_dispatch. */
MOE_API size_t moe_ep_packed_row_bytes(const moe_config* cfg);
MOE_API moe_status moe_ep_dispatch_packed(const moe_config* cfg, int n_ranks, int capacity, const int32_t* topk_idx,
                                          const float* topk_w, const void* x, int T, int32_t* send_counts,
                                          int32_t* send_tok, void* packed, moe_stream_t stream);

/* Peer-memory form of the packed dispatch: the same rows written straight into
 * every rank's receive buffer, so that no all-to-all moves them (on NVLink the
 * stores to a peer's buffer cross the link as the kernel runs).  recv_bufs is a
 * device array of n_ranks device pointers, entry q the receive buffer of rank q
 * as this process addresses it (its own buffer for q == my_rank, the peers'
 * mapped into this process, e.g. symmetric memory); each buffer holds
 * [n_ranks * capacity, moe_ep_packed_row_bytes(cfg)] bytes, 16-byte aligned.
 * Rank q's rows land in recv_bufs[q] at slots [my_rank * capacity, my_rank *
 * capacity + send_counts[q]) and the rest of those capacity slots are marked as
 * padding: after every rank has made this call, each buffer holds what
 * moe_ep_dispatch_packed plus an equal-split all-to-all would have delivered.
 * Ordering the stores before any rank reads its buffer is the caller's (a
 * collective on the stream after this call on every rank does it).
 * send_counts, send_tok and the other arguments as moe_ep_dispatch_packed;
 * 0 <= my_rank < n_ranks; recv_bufs 8-byte aligned. */
MOE_API moe_status moe_ep_dispatch_peer(const moe_config* cfg, int n_ranks, int capacity, int my_rank,
                                        const int32_t* topk_idx, const float* topk_w, const void* x, int T,
                                        int32_t* send_counts, int32_t* send_tok, void* const* recv_bufs,
                                        moe_stream_t stream);

/* Received packed rows (n_rows of them, as moe_ep_dispatch_packed lays them
 * out) into the inputs of moe_experts_routed: x_rows [n_rows, d] bf16,
 * topk_idx / topk_w [n_rows, k].  Padding rows keep ids -1 (weights 0), which
 * moe_experts_routed skips as foreign slots; their x rows are not written. */
MOE_API moe_status moe_ep_unpack(const moe_config* cfg, int n_rows, const void* packed, void* x_rows,
                                 int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Device workspace bytes of moe_experts_routed for up to n_rows_max rows and a
 * block of n_local experts (0 on invalid arguments). */
MOE_API size_t moe_experts_routed_workspace_size(const moe_config* cfg, int n_local, int n_rows_max);

/* The experts of one block on rows whose routing is given (the receiving side
 * of the dispatch; "Routed experts" and "Expert combine" boxes):
 *   y_rows[i] = routed_scale * sum over the slots j whose expert lies in
 *               [expert_lo, expert_lo + n_local) of w[i,j] * expert_{idx[i,j]}(x_rows[i])
 * fp32 [n_rows, d], overwritten; expert(x) and the arithmetic as moe_forward's.
 * w_local: the block's weights, w_gate / w_up [n_local, H, d], w_down [n_local,
 * d, H] (e4m3: with their block scales); its router and shared-expert pointers
 * are not read.  x_rows [n_rows, d] bf16; topk_idx / topk_w [n_rows, k] with
 * global expert ids (slots of other blocks are skipped, not errors).
 * workspace: moe_experts_routed_workspace_size(cfg, n_local, n_rows) bytes,
 * 256-byte aligned. */
MOE_API moe_status moe_experts_routed(const moe_config* cfg, const moe_weights* w_local, int expert_lo, int n_local,
                                      const void* x_rows, int n_rows, const int32_t* topk_idx, const float* topk_w,
                                      float* y_rows, void* workspace, size_t ws_bytes, moe_stream_t stream);

/* Combine: y_acc[send_tok[i], :] += back_rows[i, :] for i < n_rows (fp32
 * atomics: a token's partial sums from the ranks it was sent to), then, with y
 * not NULL, y = bf16(y_acc + residual) ([T, d] bf16; residual bf16 [T, d] or
 * NULL, and may be y itself).  y_acc [T, d] fp32 holds the shared expert's output
 * on entry.  A send_tok entry of -1 is a padding slot of the packed layout and
 * is skipped; any other entry outside [0, T) sets MOE_DEVERR_BAD_ROWS and its
 * row is skipped.  d a multiple of 8; arrays 16-byte aligned. */
MOE_API moe_status moe_ep_combine(int T, int d, int n_rows, const float* back_rows, const int32_t* send_tok,
                                  float* y_acc, void* y, const void* residual, moe_stream_t stream);

/* Peer-memory form of the combine for the packed layout: the partial sums of this
 * rank's slot i (i < n_ranks * capacity, send_tok as moe_ep_dispatch_peer wrote it)
 * are read straight from the result buffer of the rank that computed them,
 * result_bufs[q] + (my_rank * capacity + i % capacity) * d floats with q = i /
 * capacity (the rows moe_experts_routed wrote there over the received buffer),
 * so no all-to-all returns them; then as moe_ep_combine.  result_bufs: device
 * array of n_ranks device pointers (own buffer and mapped peers'), each
 * [n_ranks * capacity, d] fp32, 16-byte aligned; the caller orders the peers'
 * writes before this call.  capacity >= T, 0 <= my_rank < n_ranks. */
MOE_API moe_status moe_ep_combine_peer(int T, int d, int n_ranks, int capacity, int my_rank,
                                       const float* const* result_bufs, const int32_t* send_tok, float* y_acc,
                                       void* y, const void* residual, moe_stream_t stream);

/* Size of the device scratch array that moe_forward_noalloc uses in place of
 * a caller-provided workspace: 32 MiB.  At the DeepSeek-V3 sizes (d = 7168,
 * 256 experts, top-8, H = Hs = 2048, one shared expert) that holds up to
 * T = 158 tokens, which covers decode batches. */
#define MOE_NOALLOC_MAX_BYTES ((size_t)32 << 20)

/* moe_forward without a workspace argument, for callers that cannot allocate
 * device memory when they call the layer: for example code that must not
 * touch the device allocator on its path (cudaMalloc and cudaFree may
 * synchronise the whole device), or a host that embeds the layer while all
 * device memory belongs to another program's allocator with no handle it can
 * lend.  This entry point has no counterpart on the pages; it is a
 * deployment convenience around moe_forward.
 *
 *   - The scratch is one static device array of MOE_NOALLOC_MAX_BYTES per GPU
 *     that loads the library; it stays allocated until the process exits.
 *     The call allocates nothing (no cudaMalloc, cudaFree or allocating
 *     library routine).
 *   - If moe_workspace_size(cfg, T) exceeds MOE_NOALLOC_MAX_BYTES the call
 *     returns MOE_ERR_WORKSPACE and enqueues nothing; use moe_forward then.
 *   - The first call on a device looks up the array's device address for that
 *     device (cudaGetSymbolAddress, once per device, with the device current).
 *     With CUDA's lazy module loading (the default since CUDA 12.2) that first
 *     lookup is also what loads the library's device code on the device and
 *     reserves the array, which goes through the driver's allocator and may
 *     synchronise.  So make one warm-up call per device at initialisation,
 *     before any stream capture and before the path that must not allocate;
 *     later calls reserve nothing.
 *   - A device that is not sm_100 returns MOE_ERR_UNSUPPORTED, as for every
 *     other entry point.
 *   - Every call on a device shares the one array.  Calls whose work overlaps
 *     on the GPU (other streams, other host threads) race on it and give wrong
 *     results: order them on one stream or serialise them.  Whatever a
 *     previous call left in the array does not change a later call's result:
 *     every value that reaches the output is rewritten or cleared first.
 * Arguments, layouts and results as moe_forward. */
MOE_API moe_status moe_forward_noalloc(const moe_config* cfg, const moe_weights* w, const void* x,
                                       const float* bias, int T, void* y, moe_dtype y_dtype, int accumulate,
                                       moe_stream_t stream);

/* Reads and clears the calling thread's current device's error word.  This
 * call synchronises `stream` (it waits for the work enqueued before it).
 * *flags receives the MOE_DEVERR_* bits; returns MOE_ERR_DEVICE if any is set. */
MOE_API moe_status moe_device_error(unsigned int* flags, moe_stream_t stream);

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status s);

/* MOE_ABI_VERSION of the loaded library. */
MOE_API int moe_abi_version(void);

/* ---- Checking build ------------------------------------------------------
 * The library also comes as libmoe_b200_debug.so, the same sources compiled
 * with MOE_DEBUG.  Its kernels check, before every access that depends on a
 * device-built table, that the access stays inside its buffer: the permuted
 * row each token is copied to, the token of each row the combine adds into
 * y, the row count and the row range of every grouped-GEMM work item against
 * the permuted buffers and against the group's item count, and each item's
 * weight tile against the expert's weight matrix (so every TMA coordinate
 * lies inside its tensor map).  A failed
 * check sets MOE_DEVERR_BOUNDS and skips the access, or replaces the work
 * item with an in-bounds one whose output is discarded as wrong; nothing
 * traps.  It stands in for a memory checker, at the cost of a few
 * instructions per table read.  The pages have no counterpart: this is
 * build tooling around the layer. */

/* 1 in the checking build, 0 in the regular one. */
MOE_API int moe_debug_build(void);

#define MOE_DEBUG_TABLE_ROW_TOK 0   /* token of permuted row `index`: [n_rows] int32 */
#define MOE_DEBUG_TABLE_ROW_OFF 1   /* first permuted row of group `index`: [groups + 1] int32 */

/* Checking build only, for tests of the checks: arms a one-shot change of the
 * next moe_forward / moe_forward_ex call (in any thread), which after its
 * permutation writes `value` into entry `index` of the named device table,
 * as a corrupted table would hold it.  An index outside the table leaves it
 * unchanged.  table = -1 disarms.  Returns MOE_ERR_UNSUPPORTED in the regular
 * build and MOE_ERR_INVALID_ARG for an unknown table; touches no device. */
MOE_API moe_status moe_debug_corrupt_next(int table, int index, int value);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
