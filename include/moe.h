/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts
 * feed-forward layer (forward pass).
 *
 * The layer (Mixtral-style SMoE with SwiGLU experts):
 *   logits = x Wg^T                       router, a bias-free linear layer
 *   idx    = top-k experts per token      largest logits, equal logits go to
 *                                         the lower expert index
 *   w      = softmax over the k selected logits (weights sum to 1)
 *   y_e    = W2_e (silu(W1_e x) * (W3_e x))   one SwiGLU expert
 *   out    = sum_j w_j * y_{idx_j}        gate-weighted sum in token order
 *            (+ an always-on shared expert, weight 1, in moe_forward_ex)
 * Sources: "Mistral 8x7B SMoE architecture" (jsqmd.com) sec. 3.1
 * FeedForward and sec. 3.2 Gating Network; "MoE" chapter 10 of
 * LLMs-from-scratch (theaiera.top) sec. 10.3 router/top-k, sec. 10.4
 * sparse dispatch and weighted index_add, sec. 10.5 shared expert;
 * "Mixtral and MoE architecture" (astro-blog) MixtralMoE and FeedForward
 * listings.  Dispatch is dropless: every (token, slot) pair is computed.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Shapes: T tokens, d model width, E experts, d_ff expert hidden width,
 *   k experts per token, S = T*k routed rows.  All matrices are row-major
 *   with nn.Linear's [out, in] layout:
 *     x [T,d] bf16, Wg [E,d] bf16, W1 and W3 [E,d_ff,d] bf16,
 *     W2 [E,d,d_ff] bf16, out [T,d] fp32; shared expert Ws1 and Ws3
 *     [d_ffs,d] bf16, Ws2 [d,d_ffs] bf16.
 *   bf16 values are passed as raw 16-bit patterns (moe_bf16).
 * Supported sizes: 1 <= T <= 2^24; 1 <= k <= min(E, 8); 1 <= E <= 256;
 *   d and d_ff (and d_ffs) multiples of 128 with d <= 16384 and
 *   d_ff <= 65536; S*max(d, d_ff) < 2^31.  Other sizes return
 *   MOE_ERR_UNSUPPORTED; nothing falls back to another code path.
 * Pointers: every array argument is a DEVICE pointer on the current CUDA
 *   device, 16-byte aligned (MOE_ERR_INVALID_ARG otherwise); optional
 *   arguments may be NULL where stated.
 * Ownership: the caller allocates and frees every buffer, including the
 *   workspace `ws` (at least moe_workspace_size() bytes, 256-byte aligned).
 *   The library allocates no memory in any call and keeps no pointer after
 *   it returns.
 * Asynchrony: work is enqueued on `stream` and the call returns without
 *   waiting for it; no call synchronises the host except
 *   moe_get_device_error.  Buffers must stay valid until the stream has
 *   finished the work.  Calls sharing a workspace must be ordered on one
 *   stream.
 * Co-residency: the expert kernels run one CTA (or CTA pair) per SM.  The
 *   large-batch kernel, and the bf16 decode kernel when it has at least
 *   three work units per CTA, hand out their work through a global counter,
 *   so they finish whatever number of their CTAs is resident at a time.  The
 *   decode kernel with fewer units (one or two experts hit), the FP8 kernel
 *   and moe_expert_ffn_static assign work to CTAs statically; a CTA that
 *   waits on another CTA's results spins (bounded) on the assumption that
 *   all CTAs of the launch are resident, which holds when the layer has the
 *   GPU to itself.  If other work keeps SMs occupied for longer than the
 *   bound (2 s), the wait gives up with MOE_DEVERR_TIMEOUT_EPI.
 * Errors: arguments are checked on the host before anything is launched;
 *   the first failed check is returned and nothing is enqueued.  A failed
 *   launch returns MOE_ERR_CUDA.  Problems only the GPU can see (an
 *   inconsistent offsets array, a bounded wait that ran out) set an error
 *   word inside the workspace, readable with moe_get_device_error; each
 *   entry point that takes a workspace clears that word when it starts.
 *   No C++ exception crosses this interface.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */
typedef uint16_t moe_bf16;                /* raw bfloat16 bits */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null or misaligned pointer, negative size, k > E, ... */
    MOE_ERR_UNSUPPORTED = 2, /* valid but outside the supported sizes above */
    MOE_ERR_WORKSPACE = 3,   /* ws_bytes smaller than moe_workspace_size() */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime/driver call or a launch failed */
    MOE_ERR_DEVICE = 5,      /* the device error word is set (moe_get_device_error) */
    MOE_ERR_TIMEOUT = 6      /* a device-side bounded wait ran out */
} moe_status;

/* Device error word bits (moe_get_device_error's *code). */
#define MOE_DEVERR_TIMEOUT_TMA 0x1u  /* a pipeline wait for a tensor-memory copy ran out */
#define MOE_DEVERR_TIMEOUT_MMA 0x2u  /* a wait for tensor-core work ran out */
#define MOE_DEVERR_TIMEOUT_EPI 0x4u  /* a wait for the epilogue ran out */
#define MOE_DEVERR_OFFSETS 0x8u      /* offsets[] not non-decreasing within [0, S] */
#define MOE_DEVERR_INDEX 0x10u       /* an expert index or row index out of range */
#define MOE_DEVERR_LAYOUT 0x20u      /* a kernel found its shared memory misplaced and did nothing */
#define MOE_DEVERR_EP_COUNTS 0x40u   /* moe_ep_dispatch: counts_all disagrees with idx or overflows */

/* Bytes of workspace every entry point below needs for these shapes
 * (the largest need over all of them).  0 if the shapes are unsupported. */
MOE_API size_t moe_workspace_size(int T, int d, int E, int d_ff, int k);

/* Same, with a shared expert of hidden width d_ff_shared (0 = none). */
MOE_API size_t moe_workspace_size_ex(int T, int d, int E, int d_ff, int k, int d_ff_shared);

/* Router: logits = x Wg^T (+ router_bias), per-token top-k (ties to the
 * lower expert index), softmax over the k selected logits, and the
 * per-expert histogram.
 *   router_bias [E] fp32 or NULL: added to every token's logits before both
 *     the selection and the softmax (no bias on the pages' routers; used to
 *     build skewed loads)
 *   idx [T,k] int32 out: experts of each token, by logit descending
 *   w [T,k] fp32 out: their softmax weights (sum to 1 per token)
 *   counts [E] int32 out, or NULL: number of (token, slot) pairs routed to
 *     each expert
 * Passages: jsqmd.com sec. 3.2 (gate -> topk -> softmax over the selected
 * values); theaiera.top sec. 10.3 (weights sum to 1); torch.unique / per
 * expert token lists of sec. 10.4 become the histogram. */
MOE_API moe_status moe_route(int T, int d, int E, int k, const moe_bf16 *x, const moe_bf16 *Wg,
                     const float *router_bias, int32_t *idx, float *w, int32_t *counts,
                     void *ws, size_t ws_bytes, moe_stream_t stream);

/* Dispatch: group the S = T*k (token, slot) pairs by expert.
 *   idx [T,k] int32 in: experts per token (values in [0,E), distinct per token)
 *   offsets [E+1] int32 out: exclusive prefix sum of the per-expert counts;
 *     expert e owns rows offsets[e] .. offsets[e+1]-1 of x_perm
 *   row_of_slot [T,k] int32 out: the x_perm row that holds (token t, slot j)
 *   x_perm [S,d] bf16 out: x_perm[row_of_slot[t,j]] = x[t]
 * Within an expert's rows the order is by token index (stable), so the
 * result is deterministic.  An index outside [0,E), or an expert repeated
 * within a token, sets MOE_DEVERR_INDEX and that pair is skipped (its
 * row_of_slot entry is -1).  Passage: theaiera.top sec. 10.4 (mask,
 * nonzero and index_select per expert). */
MOE_API moe_status moe_permute(int T, int d, int E, int k, const moe_bf16 *x, const int32_t *idx,
                       int32_t *offsets, int32_t *row_of_slot, moe_bf16 *x_perm, void *ws,
                       size_t ws_bytes, moe_stream_t stream);

/* Experts: for every expert e and row r in [offsets[e], offsets[e+1]):
 *   y_perm[r] = W2_e (silu(W1_e x_perm[r]) * (W3_e x_perm[r]))
 *   S: rows of x_perm and y_perm; offsets [E+1] int32 (device) as returned
 *   by moe_permute; y_perm [S,d] fp32 out.  H = silu(.)*(.) is rounded to
 *   bf16 between the two products.
 * An offsets array that is not non-decreasing within [0,S] sets
 * MOE_DEVERR_OFFSETS and no row is computed.  Passages: jsqmd.com sec. 3.1
 * FeedForward; theaiera.top sec. 10.4 (fc1/fc2/fc3 of the selected rows). */
MOE_API moe_status moe_expert_ffn(int S, int d, int E, int d_ff, const moe_bf16 *x_perm,
                          const int32_t *offsets, const moe_bf16 *W1, const moe_bf16 *W3,
                          const moe_bf16 *W2, float *y_perm, void *ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Combine: out[t] = sum_{j<k} w[t,j] * y_perm[row_of_slot[t,j]]
 * (+ shared_y[t]), summed in slot order j = 0..k-1.
 *   y_perm [T*k, d] fp32, row_of_slot [T,k] int32, w [T,k] fp32,
 *   shared_y [T,d] fp32 or NULL, out [T,d] fp32 out (overwritten).
 * Passages: theaiera.top sec. 10.4 (weighted index_add back to token order)
 * and sec. 10.5 (shared expert added). */
MOE_API moe_status moe_combine(int T, int d, int k, const float *y_perm, const int32_t *row_of_slot,
                       const float *w, const float *shared_y, float *out, moe_stream_t stream);

/* The whole layer: route, dispatch, experts and combine in one call.
 * out [T,d] fp32 out.  Equivalent to moe_route + moe_permute +
 * moe_expert_ffn + moe_combine, without leaving the GPU and without any
 * host synchronisation (the call can be captured in a CUDA graph).  For
 * d <= 1024 the dispatch inside the call does not build a permuted copy of x:
 * the router gives every expert its token list and the expert kernel reads
 * the rows of x through it; the rows of an expert are then not in token
 * order inside the workspace, which does not change out (each row's expert
 * output does not depend on its position; slots are summed in order).  For
 * d > 1024 with k <= 2, no shared expert and segments large enough for the
 * CTA-pair expert kernel (prefill), the combine runs inside that kernel: its
 * down units add w[t,j] * y into out[t], which the dispatch zeroed first.
 * At most two terms reach an element and two terms added onto zero give the
 * same sum in either order, so out is still the same from run to run (it
 * may differ in the last bit from moe_combine's fused multiply-add).  Other
 * layers on that kernel (k > 2, or a shared expert) keep its per-slot rows,
 * and the shared expert's rows, as bf16 in the workspace for the combine:
 * each row is rounded once, as the hidden activations H are, which is where
 * the result can differ from the composition of the separate calls (whose
 * y_perm is fp32). */
MOE_API moe_status moe_forward(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                       const moe_bf16 *Wg, const moe_bf16 *W1, const moe_bf16 *W3,
                       const moe_bf16 *W2, float *out, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_forward with an optional router bias (see moe_route) and an optional
 * shared expert of hidden width d_ff_shared (0 = none; Ws1/Ws3/Ws2 may then
 * be NULL), whose output is added to every token with weight 1
 * (theaiera.top sec. 10.5).  The workspace must hold
 * moe_workspace_size_ex(..., d_ff_shared) bytes.  The shared expert needs
 * no routing, so it runs on a second stream of the library's own (one per
 * device, created on first use, non-blocking): the call records an event on
 * `stream`, the second stream waits for it, and `stream` waits for the
 * second stream's event before the combine.  Everything stays ordered with
 * `stream`, and the call can be captured into a CUDA graph (the fork and
 * join are captured with it).  The second stream is not valid after
 * cudaDeviceReset in the same process. */
MOE_API moe_status moe_forward_ex(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                          const moe_bf16 *Wg, const float *router_bias, const moe_bf16 *W1,
                          const moe_bf16 *W3, const moe_bf16 *W2, int d_ff_shared,
                          const moe_bf16 *Ws1, const moe_bf16 *Ws3, const moe_bf16 *Ws2,
                          float *out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Layer variants the pages describe beside the method.  All fields zero is
 * the method itself (moe_forward_ex).
 *   weights: gate-weight rule of the k selected experts
 *     MOE_WEIGHTS_SOFTMAX_TOPK  softmax over the k selected logits (the method)
 *     MOE_WEIGHTS_SOFTMAX_ALL   softmax over all E logits; the selected keep
 *                               their probabilities, not renormalised
 *                               ("Mixtral 8x7B模型架构解析" (bjdmk.com.cn),
 *                               Router.forward)
 *     MOE_WEIGHTS_SIGMOID       the logistic sigmoid of each selected logit
 *                               ("万亿 MoE" (m.xxqk.cn) forward listing)
 *     MOE_WEIGHTS_ENTROPY       entropy-controlled k ("Mixtral 8x7B模型架构解析",
 *                               routing-strategy section, entropy_aware_routing):
 *                               p = softmax(logits / 0.1) over all E; a token
 *                               keeps its top k experts when the entropy
 *                               -sum p ln p exceeds 0.8, else its top k - 1,
 *                               weighted by their p (not renormalised).  An
 *                               unused slot holds expert -1 and weight 0 (in
 *                               moe_route_variant's idx and w too) and has no
 *                               row.  Needs k >= 2; not combined with a
 *                               capacity (MOE_ERR_UNSUPPORTED).  The decision
 *                               is taken in fp32.
 *   activation: expert hidden units
 *     MOE_ACT_SILU     silu(W1 x) * (W3 x), SwiGLU (the method)
 *     MOE_ACT_SIGMOID  sigmoid(W1 x) * (W3 x), the listing's a * sigmoid(g)
 *                      with its gate g the W1 rows and a the W3 rows
 *   capacity_factor: 0 = dropless (the method); > 0: expert capacity
 *     C = floor(capacity_factor * T * k / E) ("Mistral 8x7B SMoE" (jsqmd.com)
 *     sec. 2.4, capacity factor 1.2): of the (token, slot) pairs routed to an
 *     expert only the first C in token order are computed; a dropped pair
 *     adds nothing to its token (the other slots keep their weights).
 *     Negative or non-finite values are MOE_ERR_INVALID_ARG.
 * Selection (top-k, ties to the lower index) is the same under every rule
 * (the entropy rule may drop the k-th). */
#define MOE_WEIGHTS_SOFTMAX_TOPK 0
#define MOE_WEIGHTS_SOFTMAX_ALL 1
#define MOE_WEIGHTS_SIGMOID 2
#define MOE_WEIGHTS_ENTROPY 3
#define MOE_ACT_SILU 0
#define MOE_ACT_SIGMOID 1

typedef struct {
    int weights;
    int activation;
    double capacity_factor;
} moe_variant;

/* moe_forward_ex under a layer variant (variant NULL: the method).  Same
 * workspace as moe_forward_ex. */
MOE_API moe_status moe_forward_variant(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                                       const moe_bf16 *Wg, const float *router_bias,
                                       const moe_bf16 *W1, const moe_bf16 *W3, const moe_bf16 *W2,
                                       int d_ff_shared, const moe_bf16 *Ws1, const moe_bf16 *Ws3,
                                       const moe_bf16 *Ws2, const moe_variant *variant, float *out,
                                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_route with the gate-weight rule `weights` (MOE_WEIGHTS_*). */
MOE_API moe_status moe_route_variant(int T, int d, int E, int k, const moe_bf16 *x,
                                     const moe_bf16 *Wg, const float *router_bias, int weights,
                                     int32_t *idx, float *w, int32_t *counts, void *ws,
                                     size_t ws_bytes, moe_stream_t stream);

/* The whole layer with FP8 expert weights ("Mistral 8x7B SMoE" (jsqmd.com)
 * deployment section: quantised experts, the router kept in higher
 * precision).  Each expert weight is an e4m3 code (OCP 8-bit floating point
 * E4M3, no infinities; raw bytes) times an fp32 scale of its row:
 *   W1[e,f,i] = s1[e,f] * e4m3(W1q[e,f,i])   W1q, W3q [E,d_ff,d], s1, s3 [E,d_ff]
 *   W2[e,o,f] = s2[e,o] * e4m3(W2q[e,o,f])   W2q [E,d,d_ff], s2 [E,d]
 * x, Wg and router_bias are those of moe_forward_ex (bf16 router).  Inside,
 * the token rows given to the experts and the hidden activations H are fp16
 * (every e4m3 value is exact in fp16; x and H must stay within +-65504).
 * No shared expert.  Same workspace as moe_forward.  Streaming half the
 * weight bytes of bf16 is what this path is for: decode-sized batches,
 * where the layer is bound by HBM bandwidth. */
MOE_API moe_status moe_forward_fp8(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                                   const moe_bf16 *Wg, const float *router_bias,
                                   const uint8_t *W1q, const float *s1, const uint8_t *W3q,
                                   const float *s3, const uint8_t *W2q, const float *s2,
                                   float *out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_expert_ffn for callers that cannot allocate device memory: the same
 * computation, arguments and results as moe_expert_ffn, minus the workspace.
 * The pages have no counterpart of this entry point; it exists for code that
 * may not call cudaMalloc (a plugin handed only its tensors by a host program
 * that owns all device memory, or a loop that must stay out of the
 * allocator), which still owns x_perm, offsets, the weights and y_perm.
 *   Its scratch (an error word, the expert kernel's readiness counters and
 *   the intermediate H [S, d_ff] bf16) lives in one fixed device array of
 *   MOE_STATIC_SCRATCH_BYTES inside the library; every GPU that loads the
 *   library keeps it until the process exits.  A call needs
 *     256 + align256(4 * (ceil(S/32) + E) * d_ff/128) + 2 * S * d_ff
 *   bytes of it (moe_expert_ffn_static_bytes); larger sizes return
 *   MOE_ERR_WORKSPACE before anything is launched.  Nothing is allocated and
 *   no allocating routine is called.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  The lookup is repeated after the device's
 *   context has changed (cudaDeviceReset).
 *   All calls share the one array: calls that may overlap on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  The array keeps the last call's contents; every call clears the
 *   error word and the counters itself.  The error word is read with
 *   moe_expert_ffn_static_error. */
#define MOE_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

MOE_API moe_status moe_expert_ffn_static(int S, int d, int E, int d_ff, const moe_bf16 *x_perm,
                                         const int32_t *offsets, const moe_bf16 *W1,
                                         const moe_bf16 *W3, const moe_bf16 *W2, float *y_perm,
                                         moe_stream_t stream);

/* Bytes of the fixed array a moe_expert_ffn_static call of these sizes needs
 * (the formula above); 0 for sizes outside the supported range.  The pages
 * have no counterpart. */
MOE_API size_t moe_expert_ffn_static_bytes(int S, int E, int d_ff);

/* Waits for `stream`, then reads the error word of the fixed array of the
 * current device (what the last moe_expert_ffn_static call on it left) into
 * *code (may be NULL).  Returns like moe_get_device_error.  Allocates
 * nothing.  The pages have no counterpart. */
MOE_API moe_status moe_expert_ffn_static_error(uint32_t *code, moe_stream_t stream);

/* Number of events moe_forward_traced records. */
#define MOE_TRACE_EVENTS 6

/* moe_forward_ex that also records caller-created CUDA events (cudaEvent_t,
 * created with timing enabled) on `stream` at the kernel boundaries, so the
 * caller can time each kernel with cudaEventElapsedTime:
 *   events[0] before the router kernel      events[3] before the shared-expert FFN
 *   events[1] before the dispatch scatter   events[4] before the combine
 *   events[2] before the expert FFN kernel  events[5] after the combine
 * (events[3] and events[4] mark the same point when there is no shared
 * expert, events[4] and events[5] when the expert kernel did the combine,
 * see moe_forward).  n_events must be MOE_TRACE_EVENTS.  While `stream` is being
 * captured into a CUDA graph the events are recorded as graph event nodes.
 * The layer's work and results are those of moe_forward_ex. */
MOE_API moe_status moe_forward_traced(int T, int d, int E, int d_ff, int k, const moe_bf16 *x,
                                      const moe_bf16 *Wg, const float *router_bias,
                                      const moe_bf16 *W1, const moe_bf16 *W3, const moe_bf16 *W2,
                                      int d_ff_shared, const moe_bf16 *Ws1, const moe_bf16 *Ws3,
                                      const moe_bf16 *Ws2, float *out, void *ws, size_t ws_bytes,
                                      moe_stream_t stream, void *const *events, int n_events);

/* moe_forward_fp8 with caller-created CUDA events recorded at the kernel
 * boundaries, with the meaning of moe_forward_traced's events (events[3] and
 * events[4] mark the same point: there is no shared expert). */
MOE_API moe_status moe_forward_fp8_traced(int T, int d, int E, int d_ff, int k,
                                          const moe_bf16 *x, const moe_bf16 *Wg,
                                          const float *router_bias, const uint8_t *W1q,
                                          const float *s1, const uint8_t *W3q, const float *s3,
                                          const uint8_t *W2q, const float *s2, float *out,
                                          void *ws, size_t ws_bytes, moe_stream_t stream,
                                          void *const *events, int n_events);

/* Waits for `stream`, then reads the device error word of workspace `ws`
 * into *code (may be NULL).  Returns MOE_OK if it is zero, MOE_ERR_TIMEOUT
 * if a timeout bit is set, MOE_ERR_DEVICE for any other bit, MOE_ERR_CUDA if
 * the wait or the read failed. */
MOE_API moe_status moe_get_device_error(const void *ws, uint32_t *code, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism over R ranks, one GPU each (R <= 8, E a multiple of R).
 * Rank q owns experts [q*E/R, (q+1)*E/R) and holds only their weights
 * (W1, W3, W2 of moe_ep_expert_ffn are that block, [E/R, ...]).  Every rank
 * keeps a receive buffer recv_x [recv_rows, d] bf16 and an output buffer
 * recv_y (fp32 [ksplit, recv_rows, d], or bf16 [recv_rows, d] where
 * moe_ep_output_bf16 allows) that every other rank can address (its
 * own allocation, mapped into the peers with moe_ipc_get_handle /
 * moe_ipc_open_handle), with recv_rows = moe_ep_recv_rows(T_max, E, k, R).
 * One layer step, on every rank, all on one stream:
 *   1. moe_route on the rank's own T <= T_max tokens: idx, w, counts[E];
 *   2. an all-gather of counts over the ranks into counts_all [R, E] (row r
 *      = rank r's counts), e.g. an NCCL all-gather on the same stream;
 *   3. moe_ep_dispatch: every (token, slot) row of x is stored straight into
 *      its expert owner's recv_x (the all-to-all and the permutation in one
 *      kernel);
 *   4. a barrier across the ranks on the stream (e.g. an NCCL all-reduce of
 *      one word), so that every row has arrived;
 *   5. moe_ep_expert_ffn on the rank's own recv_x -> recv_y;
 *   6. a barrier, so that every output row is complete;
 *   7. moe_ep_combine: each token's k expert rows are read from their
 *      owners' recv_y and summed, gate-weighted, in slot order.
 * No kernel waits for another GPU: the ordering across GPUs is that of the
 * caller's collectives in steps 2, 4 and 6, and nothing is read back to the
 * host, so the step can be captured in a CUDA graph.  Step 2 of the next
 * layer call also orders that call's stores after this call's reads.
 * Receive layout of owner q: its experts in index order; inside an expert,
 * the rows from rank 0, then rank 1, ...; inside one sender, token order.
 * out equals moe_forward's result up to the order of the fp32 additions
 * inside the expert kernels.
 * Passages: jsqmd.com, deployment section, problem 4 (experts placed on
 * several GPUs by hand to balance memory and load); theaiera.top sec. 10.4
 * (per-expert gathering and weighted index_add, here across ranks). */

/* Receive rows per rank: R * T_max * min(k, E/R) (every token of every rank
 * may reach min(k, E/R) experts of one owner); 0 if the sizes are invalid. */
MOE_API int moe_ep_recv_rows(int T_max, int E, int k, int R);

/* Workspace bytes of one rank for steps 3 and 5 (0: unsupported sizes). */
MOE_API size_t moe_ep_workspace_size(int T_max, int d, int E, int d_ff, int k, int R);

/* K splits of the down projection moe_ep_expert_ffn uses when a rank
 * expects rows_hint received rows (recv_y then holds that many partial
 * outputs per row, summed by moe_ep_combine). */
MOE_API int moe_ep_ffn_splits(int rows_hint, int d, int E_local, int d_ff);

/* Step 3 on rank `rank`.
 *   x [T,d] bf16, idx [T,k] int32 (this rank's routing), counts_all [R,E]
 *   int32 (device), recv_x: host array of R device addresses (element r =
 *   rank r's receive buffer as this GPU addresses it), recv_rows: rows of each.
 *   pos_of_slot [T,k] int32 out: the receive row of (t, j) in the owner of
 *   expert idx[t,j]; recv_offsets [E/R+1] int32 out: segment starts of this
 *   rank's experts in its own recv_x (valid once every rank's counts are in
 *   counts_all, which they are after step 2).
 * T may be 0 (a rank with no tokens in this step: x, idx and pos_of_slot
 * are then not read; it sends nothing but still gets its receive segments).
 * If counts_all's own row differs from the counts of idx, or some owner
 * would receive more than recv_rows rows, MOE_DEVERR_EP_COUNTS is set in the
 * workspace's error word, nothing is sent and pos_of_slot is all -1.  Resets
 * the error word (read with moe_get_device_error after step 5). */
MOE_API moe_status moe_ep_dispatch(int T, int d, int E, int k, int R, int rank,
                                   const moe_bf16 *x, const int32_t *idx,
                                   const int32_t *counts_all, moe_bf16 *const *recv_x,
                                   int recv_rows, int32_t *pos_of_slot, int32_t *recv_offsets,
                                   void *ws, size_t ws_bytes, moe_stream_t stream);

/* 1 when moe_ep_expert_ffn can write bf16 output rows for these sizes (the
 * expert kernel then writes complete rows, no K split), else 0.  bf16 rows
 * halve what the combine reads back over NVLink; each row is rounded once,
 * as the hidden activations are. */
MOE_API int moe_ep_output_bf16(int rows_hint, int d, int E_local, int d_ff);

/* Step 5: moe_expert_ffn over this rank's E/R experts on its receive buffer
 * (recv_rows = moe_ep_recv_rows(T_max, E, k, R) rows, segments from
 * recv_offsets).  rows_hint: rows the rank expects to receive (T*k with
 * balanced experts; it picks the kernel's tiling, not the result); ksplit must be
 * moe_ep_ffn_splits(rows_hint, d, E/R, d_ff).  y_bf16: 0, or 1 where
 * moe_ep_output_bf16 allows it.  recv_y out: [ksplit, recv_rows, d] fp32, or
 * [recv_rows, d] bf16 with y_bf16 (rows beyond the segments are not
 * written).  Keeps the error word of the step's dispatch. */
MOE_API moe_status moe_ep_expert_ffn(int T_max, int d, int E, int d_ff, int k, int R,
                                     int rows_hint, int ksplit, int y_bf16,
                                     const moe_bf16 *recv_x, const int32_t *recv_offsets,
                                     const moe_bf16 *W1, const moe_bf16 *W3, const moe_bf16 *W2,
                                     void *recv_y, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Step 7: out[t] = sum_{j<k} w[t,j] * (sum_q recv_y_o[q, pos_of_slot[t,j]])
 * (+ shared_y[t]), o = owner of idx[t,j], slots in order j = 0..k-1, the K
 * split partials q in order.  recv_y: host array of R device addresses of
 * the ranks' output buffers, fp32, or bf16 rows with y_bf16 = 1 (ksplit 1).
 * A slot with pos_of_slot -1 adds nothing.  out [T,d] fp32 (overwritten).
 * T = 0 does nothing. */
MOE_API moe_status moe_ep_combine(int T, int d, int E, int k, int R, int recv_rows, int ksplit,
                                  int y_bf16, const int32_t *idx, const int32_t *pos_of_slot,
                                  const float *w, const void *const *recv_y,
                                  const float *shared_y, float *out, moe_stream_t stream);

/* Size of an inter-process memory handle (cudaIpcMemHandle_t). */
#define MOE_IPC_HANDLE_BYTES 64

/* Handle of the device allocation that holds dev_ptr, for another process
 * on this node: handle (MOE_IPC_HANDLE_BYTES) out, *offset out = dev_ptr's
 * offset in that allocation. */
MOE_API moe_status moe_ipc_get_handle(const void *dev_ptr, void *handle, size_t *offset);

/* Maps another process's allocation into this one (peer access enabled):
 * *base out = its first byte here; add the sender's offset.  Not for a
 * handle of this process's own memory. */
MOE_API moe_status moe_ipc_open_handle(const void *handle, void **base);

/* Unmaps a base returned by moe_ipc_open_handle. */
MOE_API moe_status moe_ipc_close(void *base);

/* Failure-detection self-test: one thread waits, through the bounded wait
 * every pipeline of the library uses, for a barrier phase that nothing
 * completes.  After the wait's time bound (2 s) it sets
 * MOE_DEVERR_TIMEOUT_MMA in the error word of ws (cleared first; ws at least
 * 256 bytes) and the kernel returns; moe_get_device_error(ws) then reports
 * MOE_ERR_TIMEOUT and the context stays usable.  The pages have no
 * counterpart. */
MOE_API moe_status moe_selftest_wait_timeout(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Static description of a status code; never NULL. */
MOE_API const char *moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
