/*
 * lmoe.h -- C ABI of the B200 (sm_100a) Stable-LatentMoE layer with Quantile Balancing.
 *
 * The layer (forward pass, per token t of x[T,d]):
 *   r_t   = 1/sqrt(mean_j x_tj^2 + eps);  x_hat = g * x * r_t                      (RMSNorm)
 *   h     = x_hat W_down^T                      width d -> latent l              (width separation)
 *   s     = sigmoid(h W_router^T + c)           fp32 router scores [T,E]
 *   sel   = top-k of u = s + b                  larger u first, ties to the lower expert index
 *   g_i   = s_sel_i / sum_j s_sel_j             unbiased, renormalised gate weights
 *   o_i   = SwiGLU_{sel_i}(h)                   routed experts in width l (SwiGLU stands in for SiTU-GLU)
 *   y     = (sum_i g_i o_i) W_up^T + SwiGLU_shared(x_hat)
 * and Quantile Balancing (QB), a delayed bias update:
 *   q_e   = (1 - k/E) quantile of column e of s, from a 4096-bin histogram over [0,1]
 *   b_e  <- b_e - beta (u_e - mean_e u_e),  u_e = q_e + b_e   (quantile of the biased column;
 *                                                             LMOE_QB_LITERAL: u_e = q_e)
 * Sources: "KimiK3MoE架构轻量化复刻演示上线,12个交互模块详解StableLatentMoE设计逻辑"
 * (tech.news18a.com): Tab 1 (width separation, shared/routed dual path), Tab 2 Figure 2
 * (QB load balance, histogram quantile), Tab 3 (forward contract), Tab 5 (RMSNorm),
 * Tab 8-11 (QB: bias only reroutes, normalised weights, delayed, mean-centred, frozen at
 * inference), Tab 12 (SiTU-GLU, whose formula the page does not give).
 * "免费电子书:Pretraining a Mini Kimi K3" (g.15386.cn), capsules 20 and 25: experts as
 * batched matmuls over their tokens, no silent fallback when the dispatch buffer overflows.
 *
 * Conventions for every call:
 *  - Pointers named *_dev are CUDA device pointers; *_host are host pointers (pinned memory
 *    gives truly asynchronous copies).  The caller owns every pointer it passes.
 *  - Matrices are row-major.  Weights use the (out, in) layout of a linear layer.
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    and returns, except lmoe_create (returns after enqueuing its copies), lmoe_get_status
 *    and lmoe_destroy, which synchronise.  Calls on one handle are not thread-safe.
 *  - Calls return 0 (LMOE_OK) or a negative LMOE_E* code; nothing is thrown across the ABI.
 *    There is no fallback: a shape the kernels do not support returns LMOE_EUNSUPPORTED.
 *  - Faults found on the device (NaN score, an index out of range, a pipeline wait that gave
 *    up) set bits of a device status word that lmoe_get_status reads; no kernel traps.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define LMOE_OK 0
#define LMOE_EINVAL (-1)        /* bad argument: null pointer, shape, T > max_tokens, nbins != 4096 */
#define LMOE_ENOMEM (-2)        /* a device or pinned allocation failed */
#define LMOE_ECUDA (-3)         /* a CUDA call or kernel launch failed */
#define LMOE_EUNSUPPORTED (-4)  /* valid shape that these kernels do not implement */
#define LMOE_EDEVICE (-5)       /* not an sm_100 device */

/* lmoe_config.dtype: storage and arithmetic type of activations and of all weights except the
 * router (always fp32).  BF16 runs the GEMMs on tcgen05 tensor cores with fp32 accumulation;
 * F32 runs them on the tensor cores too, as split-precision products: each fp32 operand held as three
 * bf16 parts, six exact part products accumulated in fp32 (tf32 alone would not meet fp32 accuracy). */
#define LMOE_F32 0
#define LMOE_BF16 1

/* lmoe_config.experts: the operand format of the routed experts' two GEMMs.
 * BF16: bf16 operands, fp32 accumulation (as the rest of the layer).
 * MXFP8: block-scaled 8-bit operands on tcgen05.mma.kind::mxf8f6f4 (the pages give K3's experts
 * 4-bit weights and 8-bit activations after quantisation-aware training, "Kimi K3登顶开源第一..."
 * (cge.wang), and report FP8 at 0.19x of the bf16 replica's MFU on H200, the wink.run summary of
 * "Pretraining a Mini Kimi K3"; they fix no format, so the reading here is MXFP8): E4M3 elements
 * (round to nearest even, saturating at 448) with one power-of-two scale per 32 elements along K,
 * 2^X with X = floor(log2 max|v|) - 8 clamped to [-127, 127].  The expert weights are quantised
 * once at lmoe_create; the gathered latent rows (from the fp32 value of h) and the SwiGLU
 * activations (in the first GEMM's epilogue) in every forward; products accumulate in fp32 and
 * the expert outputs are bf16.  Needs dtype BF16 and l and h multiples of 128. */
#define LMOE_EXPERTS_BF16 0
#define LMOE_EXPERTS_MXFP8 1

/* lmoe_forward flags */
#define LMOE_RECORD_STATS 1u    /* add this forward's scores to the QB histogram and its expert
                                   loads to the load counters (training); without it the forward
                                   leaves the balancing state untouched */
#define LMOE_UPDATE_BIAS 4u     /* with LMOE_RECORD_STATS: the bias update of lmoe_qb_update, with
                                   the step and flags set by lmoe_set_update, runs inside this
                                   forward right after its routing (a parallel branch of the
                                   forward's work) on everything recorded up to and including
                                   this forward; it changes only later forwards */
#define LMOE_ASYNC_OUTPUT 8u     /* lmoe_forward_host only: the copy to y_host runs on a handle-owned
                                   stream, so the next call's forward overlaps it; y_host is valid
                                   only after lmoe_host_wait (see there) */
/* lmoe_qb_update flags */
#define LMOE_QB_LITERAL 1u      /* u_e = q_e (quantile of the unbiased column) */
#define LMOE_BIAS_SIGN 2u       /* aux-loss-free sign rule instead of QB (see lmoe_qb_update) */

/* device status bits (lmoe_get_status) */
#define LMOE_STATUS_NAN_SCORE 1u   /* a router score was NaN; it was never selected */
#define LMOE_STATUS_WATCHDOG 2u    /* a pipeline wait gave up after its time limit */
#define LMOE_STATUS_BAD_INDEX 4u   /* an expert index or permuted row was out of range */

#define LMOE_NBINS 4096

typedef struct lmoe_handle lmoe_handle;

typedef struct {
  int32_t d;          /* backbone width; multiple of 64 */
  int32_t l;          /* latent width; multiple of 64 */
  int32_t E;          /* routed experts; multiple of 64 for BF16, of 32 for F32; <= 1024 */
  int32_t k;          /* experts per token, 1 <= k <= min(E, 32) */
  int32_t h;          /* routed-expert SwiGLU hidden width; multiple of 64 */
  int32_t hs;         /* shared-expert SwiGLU hidden width; multiple of 64; 0 = no shared expert */
  int32_t dtype;      /* LMOE_F32 or LMOE_BF16 */
  int32_t nbins;      /* QB histogram bins; must be LMOE_NBINS */
  float rms_eps;      /* RMSNorm epsilon (1e-6) */
  int32_t max_tokens; /* largest T any forward will pass; sizes the workspace */
  int32_t experts;    /* LMOE_EXPERTS_BF16 or LMOE_EXPERTS_MXFP8 (routed-expert operand format) */
} lmoe_config;

/* Weights, all device pointers, row-major (out, in).  "dtype" means lmoe_config.dtype.
 * They are repacked into the handle: the caller may free them once lmoe_create returned
 * and `stream` has synchronised. */
typedef struct {
  const void *rms_gain;      /* [d] dtype, or NULL for all ones */
  const void *w_down;        /* [l, d] dtype */
  const float *w_router;     /* [E, l] fp32 */
  const float *router_bias;  /* [E] fp32 column offsets c, or NULL for zeros */
  const void *w1;            /* [E, h, l] dtype, SwiGLU gate projection of each expert */
  const void *w3;            /* [E, h, l] dtype, SwiGLU linear projection */
  const void *w2;            /* [E, l, h] dtype, SwiGLU output projection */
  const void *w_up;          /* [d, l] dtype */
  const void *ws1;           /* [hs, d] dtype (ignored when hs == 0) */
  const void *ws3;           /* [hs, d] dtype */
  const void *ws2;           /* [d, hs] dtype */
} lmoe_weights;

/* Validates cfg, repacks the weights (gain folded into W_down and the shared expert, gate and
 * linear projections interleaved, [W_up | Ws2] concatenated along K), allocates the workspace
 * for max_tokens and sets b = 0 and an empty histogram.  On error *out is NULL and the device
 * memory it allocated is released. */
int lmoe_create(const lmoe_config *cfg, const lmoe_weights *w, void *stream, lmoe_handle **out);

/* Releases every device allocation of the handle (synchronises the device first). */
int lmoe_destroy(lmoe_handle *h);

/* Bytes of device memory lmoe_create allocates for cfg (repacked weights + workspace + state). */
int lmoe_workspace_bytes(const lmoe_config *cfg, size_t *bytes);

/* One forward pass: y_dev[T,d] (dtype) from x_dev[T,d] (dtype), 0 <= T <= max_tokens.
 * T == 0 is a no-op.  x and y must not overlap and must be 16-byte aligned.  With
 * LMOE_RECORD_STATS the scores are added to the QB histogram and T to its token count. */
int lmoe_forward(lmoe_handle *h, const void *x_dev, void *y_dev, int32_t T, uint32_t flags,
                 void *stream);

/* The same forward with host buffers: copies x_host to the device, runs lmoe_forward into a
 * handle-owned buffer and copies the result to y_host.  The forward and the copy to y_host are
 * enqueued on `stream`; the copy from x_host runs on a handle-owned copy stream into one of two
 * staging buffers (ordered by events: it waits for the forward that last read that buffer, and
 * the forward waits for it), so one call's input copy overlaps the previous call's forward.
 * y_host is valid, and x_host may change, after `stream` synchronises.  Under stream capture of
 * `stream` everything stays on `stream`; that form is LMOE_EINVAL while the handle still counts
 * an LMOE_ASYNC_OUTPUT copy as outstanding, which lasts until a later uncaptured host-buffer
 * forward into the same staging buffer (the two buffers alternate, so the second call after it)
 * has been ordered after that copy.
 * With LMOE_ASYNC_OUTPUT the forward writes one of two handle-owned output buffers and the copy
 * to y_host runs on a second handle-owned copy stream once the forward is done; `stream` does not
 * wait for it, so a serving loop overlaps the output copy of call i with the input copy and
 * forward of call i+1 (a forward into a buffer waits for the copy that last read it).  y_host must
 * then stay allocated and unread until lmoe_host_wait has been enqueued on a stream and that
 * stream has synchronised; x_host may change after `stream` synchronises, as above. */
int lmoe_forward_host(lmoe_handle *h, const void *x_host, void *y_host, int32_t T,
                      uint32_t flags, void *stream);

/* Makes `stream` wait for every LMOE_ASYNC_OUTPUT output copy enqueued so far (they run in call
 * order on one stream).  After `stream` synchronises, every such y_host holds its forward's
 * output.  A no-op when there are none. */
int lmoe_host_wait(lmoe_handle *h, void *stream);

/* Bias update from everything recorded since the last update (N = the sum of T of those
 * forwards).  Default, Quantile Balancing: m = ceil((E-k) N / E) (exact integer), q_e = histogram
 * estimate of the m-th smallest score of expert e, b updated as above with step `beta`.
 * With LMOE_BIAS_SIGN, the aux-loss-free sign rule of "Pretraining a Mini Kimi K3" (g.15386.cn),
 * capsule 16: b_e <- b_e + beta * sign(mean_e' load_e' - load_e), load_e = (token, slot) pairs
 * routed to expert e by the recorded forwards (that page's step is beta = 1e-2); the sign is
 * decided in exact integers and the fp32 add is rounded once.  LMOE_QB_LITERAL together with
 * LMOE_BIAS_SIGN is LMOE_EINVAL.  Either rule then clears the histogram, N and the loads.
 * With N == 0 the bias is left unchanged.  Delayed: it changes only later forwards. */
int lmoe_qb_update(lmoe_handle *h, float beta, uint32_t flags, void *stream);

/* Step and flags (LMOE_QB_LITERAL or LMOE_BIAS_SIGN, as for lmoe_qb_update) of the update that
 * forwards with LMOE_UPDATE_BIAS run.  LMOE_EINVAL for a NaN step or both flags.  A forward with
 * LMOE_UPDATE_BIAS before any lmoe_set_update, or without LMOE_RECORD_STATS, is LMOE_EINVAL.
 * The result equals lmoe_forward with LMOE_RECORD_STATS followed by lmoe_qb_update on the same
 * stream: the update reads only statistics that are final once routing is done, and nothing
 * later in the forward reads the bias or the statistics. */
int lmoe_set_update(lmoe_handle *h, float beta, uint32_t flags);

/* Routing stage on caller-given scores: runs biased top-k, gates, counts, offsets, the stable
 * permutation and (with LMOE_RECORD_STATS) the histogram on scores_dev[T,E] fp32, exactly as
 * lmoe_forward does after its router.  For stage-level checks. */
int lmoe_route_scores(lmoe_handle *h, const float *scores_dev, int32_t T, uint32_t flags,
                      void *stream);

/* Copies the last forward's routing into caller buffers (any may be NULL), all device:
 *  idx [T,k] int32 (rank order), gates [T,k] fp32, scores [T,E] fp32, counts [E] int32,
 *  offsets [E+1] int32, perm [T*k] int32 (permuted row -> token; expert ascending, then token
 *  ascending), inv [T*k] int32 ((token, slot) -> permuted row). */
int lmoe_get_routing(lmoe_handle *h, int32_t *idx, float *gates, float *scores, int32_t *counts,
                     int32_t *offsets, int32_t *perm, int32_t *inv, void *stream);

/* QB state: bias b [E] fp32 (device), histogram [E, 4096] uint32 and token count N (int64),
 * all device pointers.  The scores of the last recorded forward are kept as per-score bins and
 * counted by the next lmoe_qb_update directly; lmoe_get_hist (and a second recorded forward)
 * first adds them to the histogram, so what it returns always covers every recorded forward.
 * lmoe_set_hist replaces all statistics recorded so far. */
int lmoe_get_bias(lmoe_handle *h, float *b_dev, void *stream);
int lmoe_set_bias(lmoe_handle *h, const float *b_dev, void *stream);
int lmoe_get_hist(lmoe_handle *h, uint32_t *hist_dev, int64_t *ntok_dev, void *stream);
int lmoe_set_hist(lmoe_handle *h, const uint32_t *hist_dev, const int64_t *ntok_dev, void *stream);
/* Expert loads recorded since the last update: load [E] int64, device.  Data-parallel ranks sum
 * them (with the histogram and N) before a sign-rule update, as the same page's capsule 27
 * ("Bug 2") requires: a rank that balanced its own slice would route a token by where it ran. */
int lmoe_get_load(lmoe_handle *h, int64_t *load_dev, void *stream);
int lmoe_set_load(lmoe_handle *h, const int64_t *load_dev, void *stream);

/* Synchronises the device, then returns the status word in *status and clears it. */
int lmoe_get_status(lmoe_handle *h, uint32_t *status);

/* Measurement support.  With profiling enabled, every lmoe_forward, lmoe_route_scores and
 * lmoe_qb_update records a CUDA event on its stream before each of its stages and after the last
 * (at most 4096 calls between two reads; later calls go unrecorded).  lmoe_profile_read
 * synchronises the device, stores in ms[i] (n >= 14) the time of stage i summed over the recorded
 * calls, the number of recorded forwards in *calls, and forgets the records.  Stage i is named by
 * lmoe_stage_name(i): rms, down_proj, router, norm_down_router (the three fused, when l and E are
 * at most 256), topk, plan, gather, hist, shared_swiglu, expert_swiglu, expert_down, combine,
 * up_proj, qb_update. */
int lmoe_profile_enable(lmoe_handle *h, int32_t enable);
int lmoe_profile_read(lmoe_handle *h, float *ms, int32_t n, int32_t *calls);
const char *lmoe_stage_name(int32_t i);

/* Number of kernels the handle has launched since it was created. */
int lmoe_launch_count(lmoe_handle *h, int64_t *n);

/* Routing stage for callers that cannot allocate device memory: plug-ins whose host application
 * owns every byte of device memory and hands out only fixed buffers, code that runs inside another
 * memory manager (a caching allocator or a memory pool, which must not call back into itself), and
 * real-time loops that must not enter the driver's allocator, which can synchronise the device.
 * It needs no handle and calls no cudaMalloc, cudaFree or allocating library routine.  The pages
 * have no counterpart of this entry point.
 *
 * Computes, on scores_dev [T,E] fp32 and bias_dev [E] fp32 (device, caller-owned), the same
 * routing as lmoe_route_scores: idx [T,k] int32 (rank order), gates [T,k] fp32, counts [E] int32,
 * offsets [E+1] int32, perm [T*k] int32 (permuted row -> token), inv [T*k] int32, all device
 * buffers the caller owns.  status_dev is a caller-owned device word: the call clears it, then
 * its kernels OR in LMOE_STATUS_NAN_SCORE (a NaN score, never selected) and LMOE_STATUS_BAD_INDEX
 * (an expert index or permuted row out of range); read it after the stream synchronises.
 * 1 <= k <= E (else LMOE_EINVAL); E <= 1024 and k <= 32 (else LMOE_EUNSUPPORTED, as lmoe_create).
 * Scratch: a static device array of LMOE_NOALLOC_SCRATCH_BYTES in the library image, which needs
 *   4*T*k + 8*ceil(T/32)*E + 8*(ceil(T*k/128) + E) + 132*E bytes (each part rounded up to 256) + 256;
 *   larger sizes return LMOE_EUNSUPPORTED.  The largest T is 94,496 at E = 256, k = 6 and 28,576 at
 *   E = 896, k = 16.
 * The first call on each device takes the array's device address (cudaGetSymbolAddress); make
 * that first call before any stream capture.  All calls share the one array, which keeps the
 * last call's contents: calls whose work overlaps on the GPU (other streams, other threads)
 * race and must be serialised by the caller. */
#define LMOE_NOALLOC_SCRATCH_BYTES (8u << 20)
int lmoe_route_noalloc(const float *scores_dev, const float *bias_dev, int32_t T, int32_t E, int32_t k,
                       int32_t *idx, float *gates, int32_t *counts, int32_t *offsets, int32_t *perm,
                       int32_t *inv, uint32_t *status_dev, void *stream);

/* Failure-detection check of the bounded waits: one thread waits on an mbarrier that nothing ever
 * completes, with the same wait loop every pipeline kernel uses but a limit of limit_us
 * microseconds (1 .. 2e6); it gives up, sets LMOE_STATUS_WATCHDOG in *status_dev (device word,
 * caller-owned) and returns, leaving the context usable.  No kernel of this library traps. */
int lmoe_watchdog_selftest(uint32_t *status_dev, int32_t limit_us, void *stream);

/* Static text for a return code. */
const char *lmoe_strerror(int code);

/* Check of the tensor-core GEMM engine on its own: C[M,N] (fp32) = A[M,K] B[N,K]^T with
 * A, B bf16 device buffers, K and N multiples of 64, row pitches equal to K.  M >= 256 with N a
 * multiple of 128 runs the two-CTA (cta_group::2, 256-row tile) variant.  For tests. */
int lmoe_gemm_bf16(const void *a_dev, const void *b_dev, float *c_dev, int32_t M, int32_t N,
                   int32_t K, void *stream);

/* C = op(A) op(B)^T (fp32) on the tensor-core engine with either operand stored MN-major:
 * a_mn = 0: A is [M, K] row-major; a_mn = 1: A is stored [K, M] (the product reads A^T).
 * b_mn = 0: B is [N, K]; b_mn = 1: B is stored [K, N].  N a multiple of 64, K of 8, M of 8 when
 * a_mn.  k_split > 1 (at most ceil(K/64)) cuts K into that many ranges whose products are added
 * into C by TMA reductions (C is zeroed first; the sum order then varies between runs).  M >= 256
 * with N a multiple of 128 runs the two-CTA (256-row tile) variant.  The products of the layer
 * backward use these forms.  For tests. */
int lmoe_gemm_bf16_ex(const void *a_dev, int32_t a_mn, const void *b_dev, int32_t b_mn, float *c_dev,
                      int32_t M, int32_t N, int32_t K, int32_t k_split, void *stream);

/* ---- Layer backward (training) -------------------------------------------------------------
 * Gradients of the loss L = sum(y * dy) with respect to x and every weight, for y the layer's
 * forward ("Pretraining a Mini Kimi K3" builds the training step by hand: forward, backward,
 * optimiser; "KimiK3MoE 架构轻量化复刻演示上线", Tab 6, shows the sparse expert gradients).
 * The expert choice is piecewise constant, so no gradient flows through the top-k selection or
 * into the balancing bias b; the gate weights g_i = s_i / sum_j s_j pass theirs to the chosen
 * scores through the renormalisation, and the scores to the router logits through the sigmoid
 * (unchosen scores get none).  Each expert's weight gradient sums over the (token, slot) pairs
 * routed to it only; an expert that received none gets a zero gradient.
 * All buffers fp32 device memory in the layouts of lmoe_weights; rms_gain may be NULL. */
typedef struct {
  float *dx;          /* [T, d] dL/dx */
  float *rms_gain;    /* [d] (also when the layer has no gain tensor: the gradient at gain = 1) */
  float *w_down;      /* [l, d] */
  float *w_router;    /* [E, l] */
  float *router_bias; /* [E] column offsets c */
  float *w1;          /* [E, h, l] */
  float *w3;          /* [E, h, l] */
  float *w2;          /* [E, l, h] */
  float *w_up;        /* [d, l] */
  float *ws1;         /* [hs, d] (unused when hs == 0) */
  float *ws3;         /* [hs, d] */
  float *ws2;         /* [d, hs] */
} lmoe_grads;

/* One training step's layer work on `stream`: the forward of x [T, d] into y (exactly
 * lmoe_forward with `flags`, which may record statistics but not update the bias), then every
 * gradient of lmoe_grads for the output gradient dy [T, d] (bf16, 16-byte aligned).
 * `w` must hold the weights the handle was created from, still on the device (the backward
 * reads the caller's layouts: their transposes are read in place by MN-major tensor-core
 * operands).  BF16 layers with BF16 experts only (LMOE_EUNSUPPORTED otherwise).  Operands of
 * the backward's products are bf16 (gradients are rounded to bf16 before each product),
 * accumulation fp32.  The first call allocates the backward's workspace (about
 * max_tokens * (4 d + 8 hs + 12 l + 2 E) + rows * (10 h + 4 l + 4) bytes, rows = max_tokens k +
 * 128 E) with cudaMalloc, so make it outside any stream capture; lmoe_destroy frees it.  Outside
 * a caller's stream capture, repeated calls replay CUDA graphs the handle caches: the training
 * forward has its own (beside lmoe_forward's), the backward one keyed by x, dy, T and every
 * pointer in w and g (a call that changes any of them runs eagerly, the next identical one is
 * captured, later ones replay it).  Gradients
 * of GEMMs whose output tiles cannot fill the GPU are summed over K ranges by atomic tensor
 * reductions, so their last bits vary between runs. */
int lmoe_forward_backward(lmoe_handle *h, const lmoe_weights *w, const void *x, const void *dy, void *y,
                          int32_t T, uint32_t flags, const lmoe_grads *g, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* LMOE_H */
