/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of a Laguna-style
 * token-choice mixture-of-experts layer.
 *
 * The layer (Laguna M.1/XS.2 Technical Report summary, Key claims, report
 * §3.1; Laguna-M.1-base spec sheet, "Feed-forward" and "Mixture of experts"):
 *
 *   logits_t,e = x_t . W_r[e]  (+ b_e)            sigmoid router, scores s = sigmoid(logits)
 *   S_t        = the k experts of largest score    token-choice top-k, ties -> lower index
 *   w_t,j      = s_t,e_j / sum_j' s_t,e_j'         post-top-k normalisation
 *   E_e(x)     = W_down[e] (silu(W_gate[e] x) * (W_up[e] x))   SwiGLU, no bias
 *   y_t        = Sh(x_t) + routed_scaling_factor * sum_j w_t,j E_e_j(x_t)
 *
 * with Sh an always-on shared expert of the same SwiGLU form, and
 * routed_scaling_factor the routed-expert modulation (2.5 in XS.2, 1 in M.1).
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Pointers are caller-owned DEVICE memory unless stated otherwise; the
 *   library allocates nothing per call.  bf16 tensors are passed as `const
 *   void *` and hold IEEE bfloat16 bit patterns, row-major.
 * - Weight layouts follow nn.Linear ([out, in], so the reduction dimension
 *   is contiguous): w_router [E, d]; w_gate, w_up [E, F, d]; w_down [E, d, F];
 *   ws_gate, ws_up [Fs, d]; ws_down [d, Fs].
 * - Calls are asynchronous on `stream` (a cudaStream_t passed as void *; NULL
 *   is the legacy default stream).  No call synchronises the host except
 *   moe_read_device_status, so the sequence can be captured in a CUDA graph.
 * - Every device pointer must be 16-byte aligned.  Shape limits: d_model a
 *   multiple of 64; F and Fs multiples of 64 (Fs = 0: no shared expert);
 *   1 <= k <= min(E, 16); E <= 512.  The calls that route (moe_route*,
 *   moe_forward*) also need d_model <= 14528 when the router runs on CUDA
 *   cores (T < 1024, E not a multiple of 16 or above 256, or
 *   MOE_FLAG_ROUTER_CUDA_CORE).  Anything else returns
 *   MOE_ERR_UNSUPPORTED_SHAPE before anything is launched.
 * - T = 0 is a no-op that returns MOE_OK.
 * - Errors: argument errors return synchronously and launch nothing; a failed
 *   launch returns MOE_ERR_CUDA.  Errors found on the device (a bounded wait
 *   that gave up, an out-of-range expert index) are written to a status word
 *   at the start of the workspace; moe_read_device_status returns them.  The
 *   library never aborts, exits or traps.
 * - The workspace `ws` (size from moe_workspace_size) is scratch owned by the
 *   caller.  Calls that share a workspace must not overlap on the GPU.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,        /* NULL pointer, bad struct_size, misaligned pointer */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* dims outside the limits above */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    MOE_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = 5,     /* a device-side wait gave up (see moe_read_device_status) */
    MOE_ERR_DEVICE_BOUNDS = 6       /* a device-side index check failed (e.g. expert id >= E) */
} moe_status;

/* Layer dimensions.  Field names follow the model-config keys listed on the
 * Laguna-M.1-base spec sheet ("Mixture of experts"). */
typedef struct {
    uint32_t struct_size;            /* sizeof(moe_dims_t) */
    int32_t T;                       /* tokens in this call */
    int32_t d_model;                 /* d */
    int32_t num_experts;             /* E */
    int32_t num_experts_per_tok;     /* k */
    int32_t moe_intermediate_size;   /* F, width of one routed expert */
    int32_t shared_intermediate_size;/* Fs, width of the shared expert; 0 = none */
    float routed_scaling_factor;     /* routed-expert modulation, 2.5 for XS.2 */
    int32_t norm_topk_prob;          /* 1: w = s / sum over the selected (both models); 0: w = s */
    int32_t flags;                   /* MOE_FLAG_* below; 0 = automatic choices */
} moe_dims_t;

/* flags: force one of the two router implementations (both compute the same
 * selection rule; the choice only changes speed). */
#define MOE_FLAG_ROUTER_CUDA_CORE 1   /* fp32 FMA logits + warp-per-token top-k */
#define MOE_FLAG_ROUTER_TENSOR    2   /* tcgen05 logits + the same warp-per-token top-k */
/* The caller passes fp16 copies of the down projections (w_down_f16,
 * ws_down_f16, made once by moe_prepare_down_f16); without this flag
 * moe_forward converts them into the workspace on every call. */
#define MOE_FLAG_DOWN_F16         4
/* Engine of the expert GEMMs.  By default the gate/up GEMM runs on single
 * CTAs (M = 128 tiles) and the down GEMM on CTA pairs (clusters of two SMs,
 * M = 256 tiles) when T * k >= 256 * E (the average expert fills a 256-row
 * tile), on single CTAs otherwise; these flags force one engine for both.
 * All choices give the same results. */
#define MOE_FLAG_GEMM_SINGLE_CTA  8
#define MOE_FLAG_GEMM_PAIR        16
/* router_bias is a selection-only score bias (auxiliary-loss-free load
 * balancing, Laguna-M.1-base spec sheet, Mixture of experts, "Load balancing"):
 * the k experts are those with the largest sigmoid(logit) + bias, the weights
 * are the unbiased sigmoid scores normalised over them.  Without the flag the
 * bias is added to the logits (it then changes selection and weights alike).
 * The per-expert loads (routing counts) are what a caller's bias update uses. */
#define MOE_FLAG_BIAS_SELECTION_ONLY 32
/* Size the workspace for moe_forward_fp8 (required by it; F and Fs must be
 * multiples of 128). */
#define MOE_FLAG_FP8_EXPERTS 64
/* Combine by reduction: the down GEMM adds every scaled routed row
 * (routed_scaling_factor * w * E_e(x)) and every shared-expert row straight
 * into an fp32 accumulator row of its token (bulk reduce-adds performed at
 * L2), and a last kernel rounds the accumulator to bf16 y.  No fp16
 * contribution rows are written or read back, and the sums stay in fp32; the
 * order of a token's k + 1 additions is not fixed, so repeated runs can differ
 * in the last bits of the fp32 sum (and then, rarely, by one bf16 step of y).
 * Without the flag the combine is a separate deterministic kernel over fp16
 * contribution rows.  Not with moe_forward_fp8. */
#define MOE_FLAG_COMBINE_REDUCE 128
/* Fused expert kernel: one persistent tcgen05 kernel runs the gate/up GEMM,
 * keeps the SwiGLU activation h in tensor memory (fp16, never written to
 * device memory), runs the down GEMM with its A operand read from tensor
 * memory, and adds routed_scaling_factor * w * o (shared expert: o) into
 * fp32 token rows as MOE_FLAG_COMBINE_REDUCE does (so results are rounded as
 * with that flag).  F and Fs multiples of 128, d_model a multiple of 128; an
 * FFN wider than 512 runs in parts of at most 512 columns whose partial down
 * projections add up in the same rows.  Not with moe_forward_fp8. */
#define MOE_FLAG_FUSED_EXPERTS 256

typedef struct {
    const void *w_router;      /* [E, d] bf16 */
    const float *router_bias;  /* [E] fp32 added to the logits, or NULL */
    const void *w_gate;        /* [E, F, d] bf16 */
    const void *w_up;          /* [E, F, d] bf16 */
    const void *w_down;        /* [E, d, F] bf16 */
    const void *ws_gate;       /* [Fs, d] bf16, NULL if Fs = 0 */
    const void *ws_up;         /* [Fs, d] bf16 */
    const void *ws_down;       /* [d, Fs] bf16 */
    const void *w_down_f16;    /* [E, d, F] fp16 copy of w_down (with MOE_FLAG_DOWN_F16) */
    const void *ws_down_f16;   /* [d, Fs] fp16 copy of ws_down (with MOE_FLAG_DOWN_F16) */
} moe_weights_t;

/* FP8 copies of the expert weights (moe_prepare_fp8 writes them; caller-owned
 * device memory).  Every row of every expert matrix (one output channel) is
 * stored as e4m3 codes with one float32 scale: s = amax(|row|) / 448 (1 for
 * an all-zero row), code = e4m3(w * (1 / s)), round to nearest even,
 * saturating; every step a correctly rounded float32 operation. */
typedef struct {
    void *w_gate;     /* [E, F, d] e4m3 */
    void *w_up;       /* [E, F, d] e4m3 */
    void *w_down;     /* [E, d, F] e4m3 */
    float *s_gate;    /* [E * F] scale of each row of w_gate */
    float *s_up;      /* [E * F] */
    float *s_down;    /* [E * d] */
    void *ws_gate;    /* [Fs, d] e4m3, NULL if Fs = 0 */
    void *ws_up;      /* [Fs, d] */
    void *ws_down;    /* [d, Fs] */
    float *ss_gate;   /* [Fs] */
    float *ss_up;     /* [Fs] */
    float *ss_down;   /* [d] */
} moe_fp8_weights_t;

/* Routing outputs of moe_forward (caller-owned device memory, all required). */
typedef struct {
    int32_t *topk_idx;  /* [T, k] selected experts, descending score */
    float *topk_w;      /* [T, k] normalised weights, same order */
    int32_t *counts;    /* [E] rows per expert */
    int32_t *offsets;   /* [E + 1] exclusive prefix sum of counts */
    int32_t *perm;      /* [T * k] perm[r] = t * k + j for row r in expert order */
} moe_routing_t;

/* Bytes of scratch that moe_route / moe_permute / moe_forward need for these
 * dims (0 if the dims are invalid).  The workspace must be 256-byte aligned. */
size_t moe_workspace_size(const moe_dims_t *dims);

/* Router: sigmoid scores, top-k with ties to the lower expert index, and
 * post-top-k normalisation (Laguna M.1/XS.2 Technical Report summary, Key
 * claims, report §3.1; Laguna-M.1-base spec sheet, Mixture of experts: the
 * router score is a sigmoid, the top-k weights are renormalised).  Selection is made on the logits
 * (equivalent to selection on the scores, since the sigmoid is increasing):
 * fp32 logits, and for tokens whose k-th and (k+1)-th logits are closer than
 * 2e-4, float64 logits for the experts at that boundary.
 * x: [T, d] bf16.  router_bias may be NULL.  Outputs topk_idx [T, k] int32 and
 * topk_w [T, k] fp32, both in descending-score order. */
moe_status moe_route(const moe_dims_t *dims, const void *x, const void *w_router,
                     const float *router_bias, int32_t *topk_idx, float *topk_w,
                     void *ws, size_t ws_bytes, void *stream);

/* Expert id of a (token, slot) pair that is not routed. */
#define MOE_NOT_ROUTED (-1)

/* moe_route with a padding mask: token_mask [T] uint8 device array, 0 marks a
 * padding token, which is not routed (the Laguna training notes: padding
 * tokens are best neither routed nor load-balanced).  Its k slots get
 * topk_idx = MOE_NOT_ROUTED and topk_w = 0.  token_mask = NULL routes every
 * token (same as moe_route).  Other tokens are routed exactly as by moe_route. */
moe_status moe_route_masked(const moe_dims_t *dims, const void *x, const void *w_router,
                            const float *router_bias, const uint8_t *token_mask,
                            int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                            void *stream);

/* Expert order of the (token, slot) pairs, the layout in which tokens are
 * handed to the grouped expert GEMM (Laguna M.1/XS.2 Technical Report
 * summary, Key claims, report §3.1.2, Fig. 2: tokens copied "in expert
 * order").  counts[e] = rows of expert e; offsets = exclusive prefix sum
 * ([E + 1]); perm[r] = t * k + j, rows of one expert in ascending (t, j).
 * If x and x_perm are both non-NULL the gathered rows are also materialised:
 * x_perm[r, :] = x[perm[r] / k, :] ([T * k, d] bf16).  Pairs with expert id
 * MOE_NOT_ROUTED are left out (counts and offsets[E] cover the routed pairs;
 * perm and x_perm rows past offsets[E] are not written).  Any other expert id
 * outside [0, E) sets MOE_ERR_DEVICE_BOUNDS in the status word. */
moe_status moe_permute(const moe_dims_t *dims, const int32_t *topk_idx, int32_t *counts,
                       int32_t *offsets, int32_t *perm, const void *x, void *x_perm,
                       void *ws, size_t ws_bytes, void *stream);

/* The whole layer: route, permute, the SwiGLU experts as tcgen05 grouped
 * GEMMs (gather of the permuted rows fused into the operand load), the shared
 * expert, the routed_scaling_factor modulation and the weighted combine.
 * x: [T, d] bf16 in; y: [T, d] bf16 out.  `routing` receives the router and
 * permutation results.  Precision: all accumulation is fp32; the SwiGLU
 * activation h enters the down projection as fp16 (against an fp16 copy of
 * W_down), each scaled routed contribution and the shared output are held in
 * fp16 before the fp32 combine, and y is rounded to bf16.  A value beyond the
 * fp16 range (|v| > 65504) in h or in a contribution sets
 * MOE_ERR_DEVICE_BOUNDS in the status word. */
moe_status moe_forward(const moe_dims_t *dims, const moe_weights_t *weights, const void *x,
                       void *y, const moe_routing_t *routing, void *ws, size_t ws_bytes,
                       void *stream);

/* moe_forward with a padding mask (token_mask as in moe_route_masked, NULL =
 * none).  A padding token is not routed: it adds no rows to any expert and its
 * routed contribution is zero, so y_t = shared expert(x_t) (the shared expert
 * involves no routing and is applied to every token; zero if Fs = 0).  Other
 * tokens' outputs are those of moe_forward. */
moe_status moe_forward_masked(const moe_dims_t *dims, const moe_weights_t *weights,
                              const void *x, const uint8_t *token_mask, void *y,
                              const moe_routing_t *routing, void *ws, size_t ws_bytes,
                              void *stream);

/* One-time FP8 copies of the expert weights (bf16 `weights` in, `fp8` out;
 * every pointer of `fp8` required, shared ones only if Fs > 0; scale arrays
 * 16-byte aligned).  ws needs only 256 bytes (status header). */
moe_status moe_prepare_fp8(const moe_dims_t *dims, const moe_weights_t *weights,
                           const moe_fp8_weights_t *fp8, void *ws, size_t ws_bytes, void *stream);

/* The layer with FP8 expert weights, for weight-bandwidth-bound (decode-sized)
 * batches: routing as moe_forward (bf16 router); x is quantized per token
 * (e4m3 codes, one float32 scale per row, as the weights); both expert GEMMs
 * run on e4m3 operands (tcgen05 kind::f8f6f4, fp32 accumulation) with the
 * row and column scales applied to the accumulator; h is held in fp16 and
 * quantized per row (power-of-two row scales) before the down projection; the
 * combine is moe_forward's.
 * `weights` supplies the router (w_router, router_bias); dims->flags must
 * include MOE_FLAG_FP8_EXPERTS (workspace size).  The expert GEMMs always run
 * on single CTAs. */
moe_status moe_forward_fp8(const moe_dims_t *dims, const moe_weights_t *weights,
                           const moe_fp8_weights_t *fp8, const void *x, void *y,
                           const moe_routing_t *routing, void *ws, size_t ws_bytes, void *stream);

/* One-time preparation of the down projections for moe_forward: fp16 copies
 * w_down_f16 [E, d, F] and ws_down_f16 [d, Fs] (NULL if Fs = 0) of the bf16
 * weights, rounded to nearest even (exact for 2^-14 <= |w| <= 65504; smaller
 * values become fp16 subnormals, absolute error <= 2^-25).  A weight beyond
 * the fp16 range sets MOE_ERR_DEVICE_BOUNDS in the status word of ws (which
 * needs only moe_workspace_size's first 256 bytes here).  Pass the copies in
 * moe_weights_t together with MOE_FLAG_DOWN_F16. */
moe_status moe_prepare_down_f16(const moe_dims_t *dims, const void *w_down, const void *ws_down,
                                void *w_down_f16, void *ws_down_f16, void *ws, size_t ws_bytes,
                                void *stream);

/* Byte offset of the fp32 router logits [T, E] (bias included) that
 * moe_route and moe_forward leave in the workspace.  (For small T the
 * tensor-core router splits d into up to 4 slices; their partial logits sit
 * in the planes after this one, and the selection kernel sums them, in slice
 * order, into this plane.) */
size_t moe_logits_offset(const moe_dims_t *dims);

/* Synchronises `stream`, then returns the device-side status word of `ws`
 * (MOE_OK if no kernel reported an error) and, if site != NULL, the id of the
 * place that reported it.  The status word is cleared by each moe_route /
 * moe_permute / moe_forward call. */
moe_status moe_read_device_status(const void *ws, void *stream, int32_t *site);

/* Self-test of the device timeout path: launches one kernel that waits, with
 * a bound of `limit_us` microseconds, on a flag nothing sets; it must give up
 * and write MOE_ERR_DEVICE_TIMEOUT to the status word.  Used by the tests. */
moe_status moe_selftest_bounded_wait(void *ws, size_t ws_bytes, uint32_t limit_us, void *stream);

/* Stage timing for benchmarks: arms the NEXT moe_forward call on this host
 * thread to record events (cudaEvent_t handles passed as void *, created by
 * the caller) on its stream at the six stage boundaries: before the router,
 * before the index builder, before the gate/up GEMM, before the down GEMM,
 * before the combine, and after the combine.  Events beyond n_events are not
 * recorded.  Pass events = NULL to disarm. */
moe_status moe_profile_next_forward(void **events, int32_t n_events);

/* Size of the library's static scratch array used by moe_permute_static. */
#define MOE_STATIC_SCRATCH_BYTES (512u * 1024u)

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory (code that runs inside another runtime's memory pool, or plugins
 * whose host process owns all device memory).  The source pages describe no
 * counterpart to this entry point; it is a deployment convenience.
 * Same outputs as moe_permute without x / x_perm: counts [E], offsets [E + 1],
 * perm [T * k].  Its scratch is one static device array of
 * MOE_STATIC_SCRATCH_BYTES per GPU, held from library load to process exit.
 * With n = T * k, chunk = 4096 for n <= 4096, else the smallest of 1024,
 * 2048, 4096 with 48 * chunk >= n (4096 at most), and r(b) = b rounded up to
 * a multiple of 256, the call needs
 *   256 + r(4 * E * ceil(n / chunk)) + r(16 * (ceil(n / 128) + E))
 * bytes, which must not exceed MOE_STATIC_SCRATCH_BYTES: n up to 1,384,448 at
 * E = 256, 823,296 at E = 512.  Dims that need more return
 * MOE_ERR_UNSUPPORTED_SHAPE, and nothing is launched.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress, with that
 * device current).  Every
 * call uses the same array, so calls that overlap on the GPU (other streams,
 * or other host threads) race; serialise them.  An expert id outside [0, E)
 * is skipped on the device and is not reported by this entry point.  It
 * calls no cudaMalloc, cudaFree or allocating library routine. */
moe_status moe_permute_static(const moe_dims_t *dims, const int32_t *topk_idx, int32_t *counts,
                              int32_t *offsets, int32_t *perm, void *stream);

/* Human-readable name of a status code (static string). */
const char *moe_status_string(moe_status s);

/* Number of kernel launches the last successful call on this host thread
 * issued (for launch accounting in benchmarks). */
int32_t moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
