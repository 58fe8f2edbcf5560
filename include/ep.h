/*
 * ep.h -- C ABI of the single-GPU expert-parallel dispatch/combine path
 * (sm_100a).  Plain pointers and sizes only; no C++ or framework types.
 *
 * What it computes (the DeepEP-style dispatch/combine pair):
 *   layout    counts, offsets and the stable (token, k) -> received-row
 *             permutation from the router's top-k expert ids;
 *   dispatch  copies (bf16) or quantises (FP8 E4M3, one fp32 scale per
 *             1x128 block) each token row into the expert-contiguous
 *             received buffer, once per selected expert;
 *   combine   gathers the K expert-output rows of every token back and
 *             returns their top-k weighted sum in token order.
 * Sources: "bowenzhou.top/repos/deepep/01-overview" section 1.1 (EPBuffer
 * dispatch arguments: expert_alignment, do_expand, do_zero_padding, handle),
 * section 1.3 (golden path: dispatch returns data and a handle, combine(x,
 * handle) reverses it), section 1.4 (V1 layout tensors num_tokens_per_rank,
 * is_token_in_rank, num_tokens_per_expert); "lesson14_deepep" section 3 and
 * its practice task (dispatch queues per expert, combine weighted sum);
 * "2kiu.com/news/5702702" section 2.3 (FP8 transport); "blog.hotdry.top ...
 * deepep-expert-parallel-alltoall" buffer section (num_experts divisible by
 * the number of ranks).
 *
 * Notation: T tokens, H hidden size, E experts, R logical ranks, K top-k,
 * A expert_alignment, L = E/R experts per rank.  Expert e belongs to rank
 * e / L.  Received rows are expert-major (so rank-major), and inside an
 * expert in (token, k) order; each expert segment is padded with zero rows
 * to a multiple of A.  rows = sum_e ceil(cnt_e / A) * A <= capacity =
 * T*K + E*(A-1).
 *
 * Conventions for every entry point:
 *   - return EP_OK (0) or a negative ep_error code; nothing throws;
 *   - every device pointer is a CUDA device allocation owned by the caller
 *     (except the arrays a handle owns), contiguous, row-major, 16-byte
 *     aligned unless stated; argument errors are found on the host before
 *     any launch and leave all outputs untouched;
 *   - work is enqueued on `stream` (NULL = legacy default stream) and is
 *     asynchronous: no host synchronisation, allocation or copy happens in
 *     ep_get_layout, ep_dispatch, ep_dispatch_fp8, ep_layout_dispatch(_fp8)
 *     or ep_combine;
 *   - errors found on the device (an expert id outside [0, E), a bounded
 *     in-kernel wait that gave up) set sticky bits in the handle's status
 *     word, read with ep_get_status; outputs of that call are unspecified
 *     but no out-of-bounds access is made;
 *   - a handle may be used from one stream at a time; calls on one handle
 *     from two streams that overlap on the GPU race.
 */
#ifndef EP_B200_EP_H
#define EP_B200_EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *ep_stream_t;

/* Host-side return codes. */
enum ep_error {
    EP_OK = 0,
    EP_ERR_ARG = -1,         /* null pointer, bad size, misalignment, E % R != 0 ... */
    EP_ERR_CUDA = -2,        /* a CUDA runtime call failed (see ep_last_error) */
    EP_ERR_UNSUPPORTED = -3, /* sizes beyond the library's limits (see ep_config) */
    EP_ERR_STATE = -4,       /* handle used before ep_get_layout, or on another device */
    EP_ERR_DEVICE = -5       /* ep_get_status found device-side error bits */
};

/* Device status bits (sticky until ep_clear_status). */
#define EP_DEV_BAD_EXPERT 0x1u   /* some topk_idx entry is outside [0, E) and not -1 */
#define EP_DEV_WAIT_TIMEOUT 0x2u /* a bounded in-kernel wait gave up */
#define EP_DEV_SLOT_OVERFLOW 0x4u /* low-latency: an expert was offered more pairs than its slots */

/*
 * Problem sizes, fixed for the life of a handle.
 *   num_tokens        T >= 0 (T = 0 is an empty batch)
 *   hidden            H >= 8, H % 8 == 0; H % 128 == 0 for FP8 dispatch
 *   num_experts       1 <= E <= 1024
 *   num_ranks         1 <= R <= E, E % R == 0
 *   num_topk          1 <= K <= 64 (repeated experts in a row are allowed:
 *                     every (token, k) pair still gets its own row)
 *   expert_alignment  1 <= A <= 65536
 *   T*K + E*(A-1) must stay below 2^31.
 */
typedef struct {
    int32_t num_tokens;
    int32_t hidden;
    int32_t num_experts;
    int32_t num_ranks;
    int32_t num_topk;
    int32_t expert_alignment;
} ep_config;

/* Device arrays owned by a handle (valid until ep_handle_destroy). */
typedef struct {
    const int32_t *pos;                   /* [T, K]  received row of pair (t, k), -1 if its id was invalid */
    const int32_t *row_src;               /* [capacity] token of row r, -1 for padding (rows < rows only) */
    const int32_t *row_slot;              /* [capacity] k of row r, -1 for padding */
    const float *row_weight;              /* [capacity] topk weight of row r, 0 for padding
                                             (written only if ep_get_layout had topk_weights) */
    const int32_t *num_tokens_per_expert; /* [E] */
    const int32_t *num_tokens_per_rank;   /* [R] distinct tokens with >= 1 expert on rank r */
    const int32_t *expert_offsets;        /* [E+1] padded exclusive prefix; [E] = rows */
    const int32_t *rank_offsets;          /* [R+1] = expert_offsets[r * L] */
    const uint32_t *status;               /* device status word (EP_DEV_* bits) */
    int64_t capacity;                     /* T*K + E*(A-1) */
} ep_handle_view;

typedef struct ep_handle ep_handle;

/* Checks cfg against the limits above.  Host only, no CUDA call. */
EP_API int ep_validate_config(const ep_config *cfg);

/* Worst-case received rows T*K + E*(A-1) (size recv buffers with it);
 * a negative ep_error if cfg is invalid.  Host only. */
EP_API int64_t ep_capacity_rows(const ep_config *cfg);

/* Number of scale floats per received row for FP8 dispatch: H / 128. */
EP_API int32_t ep_scales_per_row(const ep_config *cfg);

/* FP8 scale-factor layouts (ep_set_scale_layout). */
#define EP_SCALES_ROW_MAJOR 0     /* scales[row * (H/128) + b] (default) */
#define EP_SCALES_COL_MAJOR_TMA 1 /* scales[b * ld + row], ld = capacity rounded up to 4 */

/*
 * Floats a recv_scales buffer needs for `layout`: capacity * H/128 for
 * EP_SCALES_ROW_MAJOR, (H/128) * round_up(capacity, 4) for
 * EP_SCALES_COL_MAJOR_TMA; a negative ep_error for a bad cfg or layout.
 */
EP_API int64_t ep_scale_buffer_floats(const ep_config *cfg, int32_t layout);

/*
 * Creates a handle on the current CUDA device: validates cfg and allocates
 * (cudaMalloc, once) the routing arrays of ep_handle_view plus a small
 * scratch area.  The only allocating call of this library.
 */
EP_API int ep_handle_create(const ep_config *cfg, ep_handle **out);

/* Frees the handle's device memory.  Synchronises the device first. */
EP_API int ep_handle_destroy(ep_handle *h);

/* Device pointers of the arrays the handle owns (see ep_handle_view). */
EP_API int ep_handle_get_view(const ep_handle *h, ep_handle_view *out);

/*
 * Layout: from topk_idx [T, K] int64 (and optional topk_weights [T, K]
 * fp32) fills the handle's routing arrays and, for each non-NULL pointer,
 * the caller's copy:
 *   num_tokens_per_expert [E] int32, num_tokens_per_rank [R] int32,
 *   is_token_in_rank [T, R] uint8 (0/1), expert_offsets [E+1] int32,
 *   rank_offsets [R+1] int32.
 * topk_idx/topk_weights need 8/4-byte alignment only.  One kernel launch:
 * for fewer than two tokens per SM (within the ep_set_sm_limit cap), one CTA
 * per token that counts all pairs itself; else a thread-block cluster of up
 * to 16 CTAs (at most 4096 pairs each) that exchanges its histograms in
 * distributed shared memory, or, for larger batches, a cooperative grid
 * whose one grid-wide wait is bounded (EP_DEV_WAIT_TIMEOUT).
 * Defined by: the V1 layout tensors num_tokens_per_rank, is_token_in_rank
 * and num_tokens_per_expert of bowenzhou.top "deepep/01-overview" section
 * 1.4; the per-expert queue order (tokens in order, then k) of the
 * moe_dispatch loop in the "lesson14_deepep" practice task, whose counts sum
 * to T*K (its conservation assert); expert_alignment / do_zero_padding of
 * section 1.1 of the same overview page for the padded offsets.
 * An id of -1 marks an unused top-k slot (the token selects fewer than K
 * experts): that pair gets pos = -1, no row, is not counted and adds
 * nothing in combine.  Any other id outside [0, E) also gets pos = -1 and
 * sets EP_DEV_BAD_EXPERT.
 */
EP_API int ep_get_layout(ep_handle *h, const int64_t *topk_idx, const float *topk_weights,
                         int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                         uint8_t *is_token_in_rank, int32_t *expert_offsets,
                         int32_t *rank_offsets, ep_stream_t stream);

/*
 * Launch order.  ep_dispatch, ep_dispatch_fp8, ep_combine, ep_ll_dispatch,
 * ep_ll_dispatch_fp8 and ep_ll_combine launch with programmatic stream
 * serialization: the launch may begin while the previous kernel on the
 * stream is still finishing, and the kernel waits for it (and for its writes
 * to be visible) before it reads any global memory -- only its set-up and an
 * L2 prefetch of its input run earlier.  Stream order is kept exactly as for
 * an ordinary launch; the layout kernels let such a dependent start early.
 *
 * bf16 dispatch: recv_x[pos[t,k], :] = x[t, :] for every pair, and zero
 * rows for the padding of each expert segment.  x is [T, H] bf16, recv_x is
 * [capacity, H] bf16; rows at or beyond `rows` are not written.  Uses the
 * layout last computed in h (a layout may serve any number of dispatches).
 * Defined by: do_expand (one received row per (token, expert) pair) and
 * do_zero_padding of EPBuffer.dispatch, bowenzhou.top "deepep/01-overview"
 * section 1.1; the moe_dispatch loop of the "lesson14_deepep" practice task
 * (each token row appended to the queue of each expert it selected).
 */
EP_API int ep_dispatch(const ep_handle *h, const void *x, void *recv_x, ep_stream_t stream);

/*
 * FP8 dispatch: per token and 128-column block b, amax = max|x|,
 * a = max(amax, 1e-4), codes = e4m3_rn_satfinite(x * (448 / a)) (IEEE fp32
 * divide and multiply), scale[row, b] = a / 448 (the dequantisation
 * factor: x ~ code * scale).  All K copies of a token are identical;
 * padding rows are code 0x00 with scale 0.  recv_q is [capacity, H] bytes
 * (16-byte aligned); recv_scales is fp32, 4-byte aligned, in the handle's
 * scale layout (ep_set_scale_layout; default [capacity, H/128] row-major).
 * Needs H % 128 == 0.
 * Defined by: FP8 transport with the sender quantising and the receiver
 * restoring, "2kiu.com/news/5702702" section 2.3; one scaling factor per
 * block, "m.nlpx.cn/news/135159" section 4.1.  The 1x128 block, E4M3 and
 * fp32 scale are the configuration this library targets; the 1e-4 floor and
 * the stored dequantisation factor are this library's readings of what the
 * pages leave open.
 */
EP_API int ep_dispatch_fp8(const ep_handle *h, const void *x, void *recv_q, float *recv_scales,
                           ep_stream_t stream);

/*
 * Layout and dispatch in one call: the results of ep_get_layout followed by
 * ep_dispatch (or ep_dispatch_fp8), bit for bit -- the handle's routing
 * arrays, the caller's copies of the counts and offsets (each optional, as
 * in ep_get_layout), and the received rows (or codes and scales) -- so that
 * ep_combine, and further ep_dispatch calls, work on the handle afterwards.
 * Arguments as in ep_get_layout and ep_dispatch / ep_dispatch_fp8.
 *
 * Two launches that overlap: a counts pre-pass (one CTA per 16 token chunks;
 * the last CTA to finish forms the padded offsets) and the dispatch, whose
 * CTAs take token chunks in launch order from an atomic ticket, rank their
 * chunk's pairs, and find how many pairs of each expert earlier chunks hold
 * by decoupled look-back over per-chunk counts (a published single-pass scan
 * method: Merrill and Garland, 2016) -- all before they wait for the
 * pre-pass, so the layout work overlaps it and the copy starts as soon as
 * the offsets exist.  Each look-back wait is bounded (ep_set_wait_limit;
 * EP_DEV_WAIT_TIMEOUT, outputs then unspecified).  With extra_arrivals > 0
 * set by ep_set_wait_limit, the first chunk never publishes its counts: a
 * test hook that makes the waits of the chunks after it run out.
 * A batch too small to fill the GPU (fewer than two tokens per SM, within
 * the ep_set_sm_limit cap) takes one launch instead: one CTA per token, each
 * counting all T*K pairs itself (an L2 hit after the first CTA) and scanning
 * the padded counts, so no CTA waits on another; the same outputs.  T must be
 * below 2^22 (else EP_ERR_UNSUPPORTED).
 * Defined by: the same passages as ep_get_layout and ep_dispatch (the
 * queue order of the "lesson14_deepep" moe_dispatch loop; do_expand,
 * expert_alignment and do_zero_padding of bowenzhou.top "deepep/01-overview"
 * section 1.1).
 */
EP_API int ep_layout_dispatch(ep_handle *h, const int64_t *topk_idx, const float *topk_weights, const void *x,
                              void *recv_x, int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                              uint8_t *is_token_in_rank, int32_t *expert_offsets, int32_t *rank_offsets,
                              ep_stream_t stream);
EP_API int ep_layout_dispatch_fp8(ep_handle *h, const int64_t *topk_idx, const float *topk_weights, const void *x,
                                  void *recv_q, float *recv_scales, int32_t *num_tokens_per_expert,
                                  int32_t *num_tokens_per_rank, uint8_t *is_token_in_rank, int32_t *expert_offsets,
                                  int32_t *rank_offsets, ep_stream_t stream);

/*
 * Combine: out[t, :] = bf16_rn( sum_{k=0..K-1} topk_weights[t,k] *
 * y[pos[t,k], :] ), accumulated in fp32 with fused multiply-adds in k order
 * starting from 0.  y is [capacity, H] bf16 in the received-row layout of h
 * (expert outputs), topk_weights [T, K] fp32 (4-byte aligned), out [T, H]
 * bf16.  Padding rows are never read; pairs with pos = -1 add nothing.
 * Defined by: moe_combine of the "lesson14_deepep" practice task (for each
 * token, weight * expert output added back for k = 0..K-1); combine(x,
 * handle) of the golden path, bowenzhou.top "deepep/01-overview" section 1.3.
 */
EP_API int ep_combine(const ep_handle *h, const void *y, const float *topk_weights, void *out,
                      ep_stream_t stream);

/*
 * Copies the handle's routing arrays into caller device buffers (any
 * pointer may be NULL to skip it), stream-ordered: pos [T, K] int32,
 * row_src / row_slot [capacity] int32, row_weight [capacity] fp32.  The
 * analogue of EPBuffer.dispatch's do_handle_copy (bowenzhou.top
 * "deepep/01-overview" section 1.1): the copy outlives later layouts.
 */
EP_API int ep_copy_routing(const ep_handle *h, int32_t *pos, int32_t *row_src, int32_t *row_slot,
                           float *row_weight, ep_stream_t stream);

/*
 * Layout without any allocation.  This entry point has no counterpart on the
 * pages: it exists for callers that cannot call cudaMalloc where they route
 * tokens -- code that must not trigger a device allocation (it can
 * synchronise the device or fail under memory pressure), runtimes that hand
 * out device memory only from their own pools, or callers with nowhere to
 * keep a handle.  It computes exactly what ep_get_layout computes, but every
 * output comes from the caller:
 *   pos [T, K], row_src / row_slot [capacity] int32, row_weight [capacity]
 *   fp32 (required iff topk_weights is non-NULL), num_tokens_per_expert [E],
 *   num_tokens_per_rank [R], expert_offsets [E+1], rank_offsets [R+1]
 *   (all required, 4-byte aligned); is_token_in_rank [T, R] (optional);
 *   status: one device uint32, set to 0 and then to the EP_DEV_* bits of this
 *   call (read it after the stream has reached it).
 * A batch that fits one thread-block cluster (see ep_get_layout) needs no
 * scratch.  A larger one runs the cooperative kernel, whose scratch lives in
 * a fixed 256 KiB array in the library's device code, held on every GPU that
 * loads the library until exit; one that needs more (E + R columns of
 * ceil(G/4)*4 int32, G layout CTAs ~ T*K/1024 up to the SM count, plus 256
 * bytes) is rejected with EP_ERR_UNSUPPORTED and a message in ep_last_error.
 * The first call on a device does a one-time set-up on the host (it looks up
 * the array's device address and sets a kernel attribute): make that first
 * call before any stream capture.  Every call shares the one array and
 * clears the part it uses (stream-ordered memset), so calls that overlap on
 * the GPU -- on two streams, or from two threads -- race and must not be
 * issued.  No cudaMalloc, cudaFree or other allocating call is made.
 * The set-up is kept per device for the life of the process: after a
 * cudaDeviceReset the library's device state (this set-up, kernel
 * attributes, every handle) is stale, and calls after a reset in the same
 * process are not supported.
 */
EP_API int ep_get_layout_noalloc(const ep_config *cfg, const int64_t *topk_idx, const float *topk_weights,
                                 int32_t *pos, int32_t *row_src, int32_t *row_slot, float *row_weight,
                                 int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                                 uint8_t *is_token_in_rank, int32_t *expert_offsets, int32_t *rank_offsets,
                                 uint32_t *status, ep_stream_t stream);

/*
 * Launch shape of the layout for cfg on the current device, host only (the
 * first query on a device does the same one-time set-up as the first
 * ep_get_layout_noalloc call): *cluster = 1 when one thread-block cluster
 * computes it (no scratch), 0 for the cooperative kernel; *ctas = CTAs
 * launched; *noalloc_scratch_bytes = bytes of the fixed array that
 * ep_get_layout_noalloc would use (0 for the cluster kernel; a call that
 * needs more than the array's 256 KiB is rejected).  Any pointer may be NULL.
 */
EP_API int ep_layout_shape(const ep_config *cfg, int32_t *cluster, int32_t *ctas, int64_t *noalloc_scratch_bytes);

/*
 * ---- Low-latency (static, masked) layout ----
 * The decode-time mode of lesson14_deepep (hsthanb4.github.io) section 2(1)
 * -- pre-allocated static buffers and a per-expert mask, no host
 * involvement, CUDA-graph compatible -- and its section 3 listing
 * (low_latency_dispatch returns received rows per expert plus counts that a
 * masked grouped GEMM takes as its mask; low_latency_combine takes the expert
 * outputs with topk_idx and topk_weights).  blog.hotdry.top (buffer
 * section) advises num_max_dispatch_tokens_per_rank below 256.
 *
 * Every expert e owns M = num_max_dispatch_tokens fixed received rows
 * e*M .. e*M+M-1 (capacity E*M rows).  Pair (t, k) with e = topk_idx[t,k]
 * takes slot s = #{(t', k') before (t, k) in (token, k) order with the
 * same expert}, i.e. row e*M + s, the same order as the normal layout.
 * recv_count[e] = min(pairs of e, M) is the mask: slots at or past it are
 * not written (no padding, no zero fill).  A pair past an expert's M-th
 * slot is dropped (pos = -1) and sets EP_DEV_SLOT_OVERFLOW; with distinct
 * experts per token and T <= M that cannot happen.  -1 ids are masked
 * slots; other ids outside [0, E) set EP_DEV_BAD_EXPERT.  Layout and copy
 * are one kernel launch with no grid-wide wait.
 */

/* E * M received rows for M slots per expert; negative ep_error if invalid. */
EP_API int64_t ep_ll_capacity_rows(const ep_config *cfg, int32_t num_max_dispatch_tokens);

/*
 * Floats a low-latency recv_scales buffer needs: E*M*(H/128) for
 * EP_SCALES_ROW_MAJOR; for EP_SCALES_COL_MAJOR_TMA each expert's scales are
 * [H/128][round_up(M, 4)] (one TMA-aligned block per expert), E of them.
 */
EP_API int64_t ep_ll_scale_buffer_floats(const ep_config *cfg, int32_t num_max_dispatch_tokens, int32_t layout);

/*
 * Creates a low-latency handle: T = cfg->num_tokens tokens per call with
 * T <= num_max_dispatch_tokens (else EP_ERR_ARG); cfg->expert_alignment is
 * not used.  Owns pos [T, K] and the status word (one cudaMalloc).  Works
 * with ep_ll_dispatch, ep_ll_dispatch_fp8, ep_ll_combine, ep_copy_routing
 * (pos only), ep_get_status, ep_clear_status, ep_set_sm_limit,
 * ep_set_scale_layout and ep_handle_get_view (pos, status, capacity); the
 * normal-layout calls return EP_ERR_STATE on it, and ep_ll_* calls on a
 * normal handle return EP_ERR_STATE.
 */
EP_API int ep_ll_handle_create(const ep_config *cfg, int32_t num_max_dispatch_tokens, ep_handle **out);

/*
 * Low-latency bf16 dispatch: slots from topk_idx [T, K] int64 as above,
 * recv_x[e*M + s, :] = x[t, :]; recv_count [E] int32 (NULL: skip).  x is
 * [T, H] bf16, recv_x [E*M, H] bf16 (16-byte aligned).  Also records pos in
 * the handle for ep_ll_combine.  One kernel launch.
 */
EP_API int ep_ll_dispatch(ep_handle *h, const int64_t *topk_idx, const void *x, void *recv_x,
                          int32_t *recv_count, ep_stream_t stream);

/*
 * Low-latency FP8 dispatch: the slots of ep_ll_dispatch with the
 * quantisation of ep_dispatch_fp8.  recv_q [E*M, H] bytes; recv_scales in
 * the handle's scale layout (ep_ll_scale_buffer_floats).  Needs H % 128 == 0.
 */
EP_API int ep_ll_dispatch_fp8(ep_handle *h, const int64_t *topk_idx, const void *x, void *recv_q,
                              float *recv_scales, int32_t *recv_count, ep_stream_t stream);

/*
 * Low-latency combine: out[t, :] = bf16_rn(fp32 fma chain over k of
 * topk_weights[t,k] * y[pos[t,k], :]) with the pos of the last
 * ep_ll_dispatch on h; y is [E*M, H] bf16 (expert outputs in the slots),
 * out [T, H] bf16.  Dropped and masked pairs add nothing.
 */
EP_API int ep_ll_combine(const ep_handle *h, const void *y, const float *topk_weights, void *out,
                         ep_stream_t stream);

/*
 * Expert GEMM with the combine fused into its epilogue (tcgen05 tensor
 * cores): the last linear map of each expert applied to its received rows,
 * each result row scaled by its pair's top-k weight and added into the
 * token's output row -- the step between dispatch and combine of
 * "lesson14_deepep" (practice task: experts transform the rows they
 * received, moe_combine adds weight * expert output back per token), done
 * without writing the expert outputs.
 *   out[t, :] = bf16_rn( sum_k topk_weights[t,k] * act[pos[t,k], :] @ W_e^T ),
 *   e = topk_idx[t,k]; masked (-1) pairs and padding rows add nothing.
 * act [capacity, inner] bf16 in h's received-row layout; w [E, n_out, inner]
 * bf16 (expert e's matrix, row n = output feature n); topk_weights [T, K]
 * fp32; out_acc [T, n_out] fp32 workspace (zeroed by the call); out
 * [T, n_out] bf16.  Needs expert_alignment % 128 == 0 (each 128-row tile
 * belongs to one expert), inner % 64 == 0, n_out % 256 == 0 and 16-byte
 * aligned act, w, out_acc and out; else EP_ERR_ARG.  The fp32 sums are
 * formed with atomic adds, so their order (and the last bit of out) may
 * vary between calls.  Launches the GEMM (one CTA per SM, capped by
 * ep_set_sm_limit) and a rounding kernel.
 */
EP_API int ep_expert_combine(const ep_handle *h, const void *act, int32_t inner, const void *w, int32_t n_out,
                             const float *topk_weights, float *out_acc, void *out, ep_stream_t stream);

/*
 * The same expert GEMM and fused combine with FP8 operands: the rows are the
 * E4M3 codes and fp32 dequantisation scales that ep_dispatch_fp8 writes
 * (a row restores as code * scale per 128 columns, "2kiu.com/news/5702702"
 * section 2.3), and each expert matrix is E4M3 with one fp32 scale per
 * 128 x 128 block (per-block scaling, "m.nlpx.cn/news/135159" section 4.1;
 * the grouped FP8 expert GEMM that consumes the dispatch in "lesson14_deepep"
 * section 3).
 *   out[t, n] = bf16_rn( sum_k topk_weights[t,k] * sum_i A[r,i] * W_e[n,i] ),
 *   r = pos[t,k], e = topk_idx[t,k],
 *   A[r,i] = act_q[r,i] * scale(r, i/128),  W_e[n,i] = w_q[e,n,i] * w_scales[e, n/128, i/128].
 * act_q [capacity, inner] E4M3 in h's received-row layout; act_scales in h's
 * scale layout (ep_set_scale_layout: row-major [capacity, inner/128], or
 * column-major with the TMA-aligned leading dimension), as ep_dispatch_fp8
 * writes them for hidden == inner; w_q [E, n_out, inner] E4M3; w_scales
 * [E, n_out/128, inner/128] fp32; topk_weights, out_acc and out as in
 * ep_expert_combine.  The tensor cores multiply E4M3 (tcgen05 kind::f8f6f4)
 * one 128-deep block at a time; each block's fp32 product is scaled by its
 * two scales and summed in fp32.  Needs expert_alignment % 128 == 0,
 * inner % 128 == 0, n_out % 256 == 0, 16-byte aligned act_q, w_q, out_acc and
 * out, 4-byte aligned scales; else EP_ERR_ARG.  Same ordering caveat and
 * launches as ep_expert_combine.
 */
EP_API int ep_expert_combine_fp8(const ep_handle *h, const uint8_t *act_q, const float *act_scales, int32_t inner,
                                 const uint8_t *w_q, const float *w_scales, int32_t n_out,
                                 const float *topk_weights, float *out_acc, void *out, ep_stream_t stream);

/*
 * Peer-memory exchange between the GPUs of a node.  One process per GPU, R =
 * the number of GPUs, rank r owning experts [r*L, (r+1)*L).  This is the
 * exchange step of DeepEP's normal mode done inside the kernels: tokens
 * travel over NVLink straight into the other GPUs' buffers
 * ("blog.hotdry.top ... deepep-expert-parallel-alltoall", first section;
 * "bowenzhou.top/repos/deepep/01-overview" section 1.3).
 *
 * With h's layout (num_ranks = R), the rows bound for rank r are the segment
 * [rank_offsets[r], rank_offsets[r+1]).  Rank r's receive buffer holds the
 * segments of all sources one after another (source order is the caller's
 * choice); this source's block starts at row row0[r].  Row i of the segment
 * goes to row row0[r] + i of rank r's buffer.
 *
 * ep_dispatch_peer writes each token row of x ([T, H] bf16) once per
 * selected expert directly into the destination rank's buffer, and padding
 * rows (expert_alignment > 1) as zeros.  The written bytes equal what
 * ep_dispatch writes into segment r of a local buffer.  ep_combine_peer reads
 * the expert-output rows from the same places (y_bases[r] has the row
 * layout of rank r's receive buffer) and writes
 *   out[t] = bf16_rn( sum_k topk_weights[t,k] * y[row of (t,k)] ),
 * the ep_combine result.
 *
 * recv_bases / y_bases: DEVICE array of R device pointers (8-byte aligned
 * array; each pointer 16-byte aligned), valid in this process: this GPU's own
 * buffer for its rank, ep_ipc_open_handle results for the others.  row0:
 * DEVICE array of R int32.  Each buffer must hold row0[r] + (rank_offsets[r+1]
 * - rank_offsets[r]) rows of H bf16.  These contents are not checked on the
 * host; a wrong value writes or reads outside the caller's buffers.  Null,
 * misaligned or host-detectable errors return EP_ERR_ARG; a low-latency handle
 * returns EP_ERR_STATE; an empty batch (T = 0) returns EP_OK and launches
 * nothing.  The calls issue plain loads and stores and never wait
 * on another GPU.  The caller orders the ranks: every destination buffer is
 * free before a dispatch starts, and every expert output is complete before a
 * combine reads it (for example, a stream synchronise and a process-group
 * barrier).
 */
EP_API int ep_dispatch_peer(const ep_handle *h, const void *x, void *const *recv_bases, const int32_t *row0,
                            ep_stream_t stream);
EP_API int ep_combine_peer(const ep_handle *h, const void *const *y_bases, const int32_t *row0,
                           const float *topk_weights, void *out, ep_stream_t stream);

/*
 * FP8 form of ep_dispatch_peer: each destination receives E4M3 codes
 * (recv_bases[r]: [rows, H] bytes) and fp32 scales (scale_bases[r]: DEVICE
 * array of R pointers, each to [rows, H/128] floats, row-major, 4-byte
 * aligned), the bytes ep_dispatch_fp8 writes into segment r of a local
 * buffer; padding rows get codes 0 and scales 0.  Needs H % 128 == 0 (else
 * EP_ERR_ARG) and the handle's row-major scale layout (else
 * EP_ERR_UNSUPPORTED).  Combine takes bf16 expert outputs, as ep_combine_peer.
 */
EP_API int ep_dispatch_peer_fp8(const ep_handle *h, const void *x, void *const *recv_bases,
                                float *const *scale_bases, const int32_t *row0, ep_stream_t stream);

/*
 * CUDA IPC for those buffers.  ep_ipc_get_handle fills `handle`
 * (EP_IPC_HANDLE_BYTES opaque bytes) for the allocation that contains
 * dev_ptr and sets *offset to dev_ptr's byte offset inside it (allocators
 * that sub-allocate return pointers inside a larger allocation).  In another
 * process, ep_ipc_open_handle maps that allocation and returns its base;
 * add the offset to reach dev_ptr.  ep_ipc_close_handle unmaps a base that
 * ep_ipc_open_handle returned.  A process cannot open its own handles.
 */
#define EP_IPC_HANDLE_BYTES 64
EP_API int ep_ipc_get_handle(const void *dev_ptr, void *handle, int64_t *offset);
EP_API int ep_ipc_open_handle(const void *handle, void **base);
EP_API int ep_ipc_close_handle(void *base);

/* Synchronises `stream` and returns rows (= expert_offsets[E]) on the host. */
EP_API int ep_get_num_rows(const ep_handle *h, int32_t *rows, ep_stream_t stream);

/*
 * Synchronises `stream` and returns the device status bits; EP_OK if they
 * are zero, EP_ERR_DEVICE otherwise.
 */
EP_API int ep_get_status(const ep_handle *h, uint32_t *bits, ep_stream_t stream);

/* Clears the status word and the in-kernel wait state (stream-ordered). */
EP_API int ep_clear_status(ep_handle *h, ep_stream_t stream);

/*
 * Layout of the scales ep_dispatch_fp8 writes on this handle (default
 * EP_SCALES_ROW_MAJOR).  EP_SCALES_COL_MAJOR_TMA stores them column-major
 * with the row dimension padded to a multiple of 4 floats, so every 1x128
 * block column starts 16-byte aligned -- the layout a grouped FP8 GEMM reads
 * with TMA (the use_tma_aligned_col_major_sf option of EPBuffer.dispatch,
 * bowenzhou.top "deepep/01-overview" section 1.1).  Values are identical in
 * both layouts; size the buffer with ep_scale_buffer_floats.
 */
EP_API int ep_set_scale_layout(ep_handle *h, int32_t layout);

/*
 * Caps the SMs that ep_dispatch, ep_dispatch_fp8 and ep_combine occupy on
 * this handle (0 = all, the default; values above the device's count mean
 * all).  Their persistent grids are sized to at most `num_sms` SMs, so the
 * rest of the GPU stays free for work that overlaps them -- the role of
 * DeepEP's num_sms argument (bowenzhou.top "deepep/01-overview" section 1.1;
 * "blog.hotdry.top ... deepep-expert-parallel-alltoall": 24 SMs by default;
 * "lesson14_deepep" section 1(2): 20 communication SMs beside 110 compute
 * SMs).  The layout kernel is not capped (it uses at most 16 CTAs, or one
 * CTA per 1024 pairs beyond that).  Results do not depend on the cap.
 */
EP_API int ep_set_sm_limit(ep_handle *h, int32_t num_sms);

/*
 * Limit for each bounded in-kernel wait, in nanoseconds of %globaltimer
 * (default 1e9).  `extra_arrivals` > 0 makes the layout's grid-wide wait
 * expect that many CTAs that never arrive, and makes the first chunk of
 * ep_layout_dispatch(_fp8) never publish its counts: test hooks that
 * exercise the timeout paths without hanging (the waits give up after
 * limit_ns and set EP_DEV_WAIT_TIMEOUT).  Use 0 in normal operation.
 */
EP_API int ep_set_wait_limit(ep_handle *h, uint64_t limit_ns, int32_t extra_arrivals);

/* Static description of a return code. */
EP_API const char *ep_status_string(int code);

/* Text of the last CUDA error seen by this library on the calling thread. */
EP_API const char *ep_last_error(void);

/* Number of kernels this library has launched in this process. */
EP_API uint64_t ep_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_H */
