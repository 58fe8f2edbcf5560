// ep_api.cu -- host side of the C ABI declared in include/ep.h.
//
// Validates arguments, owns the handle's device arrays, chooses launch
// shapes once per handle and enqueues kernels.  No host synchronisation,
// allocation or copy on the layout/dispatch/combine calls.
#include <atomic>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <new>

#include <cuda.h>

#include "ep_internal.cuh"
#include "peer.cuh"

namespace {

thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};

int cuda_fail(cudaError_t e, const char *what) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
    return EP_ERR_CUDA;
}

#define EP_CUDA(call)                                               \
    do {                                                            \
        cudaError_t _e = (call);                                    \
        if (_e != cudaSuccess) return cuda_fail(_e, #call);         \
    } while (0)

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Makes the handle's device current for the duration of a call.
struct DeviceGuard {
    int prev = -1;
    cudaError_t err = cudaSuccess;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) err = cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

int check_handle(const ep_handle *h, bool need_layout) {
    if (!h) return EP_ERR_ARG;
    if (need_layout && !h->has_layout) return EP_ERR_STATE;
    return EP_OK;
}

// Calls of one layout mode on a handle of the other return EP_ERR_STATE.
int check_mode(const ep_handle *h, bool ll, bool need_layout) {
    int rc = check_handle(h, false);
    if (rc != EP_OK) return rc;
    if ((h->ll_M > 0) != ll) return EP_ERR_STATE;
    return check_handle(h, need_layout);
}

}  // namespace

namespace ep {
void record_error(const char *msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }
int record_cuda_error(cudaError_t e, const char *what) { return cuda_fail(e, what); }
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace ep

extern "C" {

EP_API int ep_validate_config(const ep_config *c) {
    if (!c) return EP_ERR_ARG;
    if (c->num_tokens < 0 || c->hidden < 8 || c->hidden % 8 != 0) return EP_ERR_ARG;
    if (c->num_experts < 1 || c->num_ranks < 1 || c->num_ranks > c->num_experts) return EP_ERR_ARG;
    if (c->num_experts % c->num_ranks != 0) return EP_ERR_ARG;
    if (c->num_topk < 1 || c->expert_alignment < 1) return EP_ERR_ARG;
    if (c->num_experts > ep::kMaxExperts || c->num_topk > ep::kMaxTopk || c->expert_alignment > 65536)
        return EP_ERR_UNSUPPORTED;
    const int64_t cap = (int64_t)c->num_tokens * c->num_topk +
                        (int64_t)c->num_experts * (c->expert_alignment - 1);
    if (cap >= (int64_t(1) << 31)) return EP_ERR_UNSUPPORTED;
    return EP_OK;
}

EP_API int64_t ep_capacity_rows(const ep_config *c) {
    const int rc = ep_validate_config(c);
    if (rc != EP_OK) return rc;
    return (int64_t)c->num_tokens * c->num_topk + (int64_t)c->num_experts * (c->expert_alignment - 1);
}

EP_API int32_t ep_scales_per_row(const ep_config *c) {
    const int rc = ep_validate_config(c);
    if (rc != EP_OK) return rc;
    return c->hidden / 128;
}

EP_API int64_t ep_scale_buffer_floats(const ep_config *c, int32_t layout) {
    const int64_t cap = ep_capacity_rows(c);
    if (cap < 0) return cap;
    if (c->hidden % 128 != 0) return EP_ERR_ARG;
    const int64_t nb = c->hidden / 128;
    if (layout == EP_SCALES_ROW_MAJOR) return cap * nb;
    if (layout == EP_SCALES_COL_MAJOR_TMA) return nb * ((cap + 3) / 4 * 4);
    return EP_ERR_ARG;
}

EP_API int ep_handle_create(const ep_config *cfg, ep_handle **out) {
    if (!out) return EP_ERR_ARG;
    *out = nullptr;
    int rc = ep_validate_config(cfg);
    if (rc != EP_OK) return rc;

    ep_handle *h = new (std::nothrow) ep_handle();
    if (!h) return EP_ERR_ARG;
    h->cfg = *cfg;
    h->cap = ep_capacity_rows(cfg);
    h->wait_limit_ns = ep::kDefaultWaitLimitNs;
    h->barrier_extra = 0;
    h->has_layout = false;
    h->sm_limit = 0;
    h->scale_layout = EP_SCALES_ROW_MAJOR;
    h->ll_M = 0;

    auto fail = [&](int code) {
        delete h;
        return code;
    };
    cudaError_t e = cudaGetDevice(&h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaGetDevice"));
    e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaDeviceGetAttribute"));
    e = cudaDeviceGetAttribute(&h->l2_bytes, cudaDevAttrL2CacheSize, h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaDeviceGetAttribute(L2)"));

    const int T = cfg->num_tokens, E = cfg->num_experts, R = cfg->num_ranks, K = cfg->num_topk;

    // layout launch shape (cluster kernel, or the cooperative fallback)
    e = ep::layout_prepare(h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "layout set-up"));
    h->plan = ep::plan_layout(h->device, T, E, R, K, h->num_sms);
    if (!h->plan.cluster) {
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ep::layout_kernel_ptr(), ep::kLayoutThreads,
                                                          h->plan.smem);
        if (e != cudaSuccess) return fail(cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor"));
        if (per_sm < 1) return fail(EP_ERR_UNSUPPORTED);
    }
    const int64_t G = h->plan.G;
    h->G = h->plan.G;
    h->tokens_per_chunk = h->plan.tokens_per_chunk;

    e = ep::dispatch_lb_prepare();
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaFuncSetAttribute(dispatch)"));
    h->lb = ep::plan_lb(T, K, h->num_sms);

    // carve one allocation
    const size_t A256 = 256;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + (bytes ? bytes : 1), A256);
        return o;
    };
    const size_t o_pos = take(sizeof(int32_t) * (size_t)T * K);
    const size_t o_src = take(sizeof(int32_t) * (size_t)h->cap);
    const size_t o_slot = take(sizeof(int32_t) * (size_t)h->cap);
    const size_t o_w = take(sizeof(float) * (size_t)h->cap);
    const size_t o_cnt = take(sizeof(int32_t) * E);
    const size_t o_rtok = take(sizeof(int32_t) * R);
    const size_t o_eoff = take(sizeof(int32_t) * (E + 1));
    const size_t o_roff = take(sizeof(int32_t) * (R + 1));
    // chunk histograms of the cooperative kernel (the cluster kernel needs none)
    const size_t o_chunk = take(h->plan.cluster ? 0 : sizeof(int32_t) * (size_t)((G + 3) / 4 * 4) * (E + R));
    const size_t o_bar = take(sizeof(ep::GridBarrier));
    const size_t o_stat = take(sizeof(unsigned int));
    // the fused layout + dispatch: control words, super-chunk histograms and
    // bases, look-back words
    const size_t o_lbctl = take(sizeof(ep::LbControl));
    const size_t o_lbhist = take(sizeof(int32_t) * (size_t)h->lb.nsuper * (E + R));
    const size_t o_lbbase = take(sizeof(int32_t) * (size_t)h->lb.nsuper * E);
    const size_t o_lbflags = take(sizeof(unsigned long long) * (size_t)h->lb.nchunks * E);
    const size_t o_lbready = take(sizeof(unsigned int) * (size_t)h->lb.nchunks);
    h->block_bytes = off;
    e = cudaMalloc(&h->block, h->block_bytes);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaMalloc(handle)"));
    e = cudaMemset(h->block, 0, h->block_bytes);
    if (e != cudaSuccess) {
        cudaFree(h->block);
        return fail(cuda_fail(e, "cudaMemset(handle)"));
    }
    char *b = static_cast<char *>(h->block);
    h->pos = reinterpret_cast<int32_t *>(b + o_pos);
    h->row_src = reinterpret_cast<int32_t *>(b + o_src);
    h->row_slot = reinterpret_cast<int32_t *>(b + o_slot);
    h->row_weight = reinterpret_cast<float *>(b + o_w);
    h->cnt = reinterpret_cast<int32_t *>(b + o_cnt);
    h->rank_tok = reinterpret_cast<int32_t *>(b + o_rtok);
    h->eoff = reinterpret_cast<int32_t *>(b + o_eoff);
    h->roff = reinterpret_cast<int32_t *>(b + o_roff);
    h->chunk_counts = reinterpret_cast<int32_t *>(b + o_chunk);
    h->barrier = reinterpret_cast<ep::GridBarrier *>(b + o_bar);
    h->status = reinterpret_cast<unsigned int *>(b + o_stat);
    h->lb_ctl = reinterpret_cast<ep::LbControl *>(b + o_lbctl);
    h->lb_super_hist = reinterpret_cast<int32_t *>(b + o_lbhist);
    h->lb_super_base = reinterpret_cast<int32_t *>(b + o_lbbase);
    h->lb_flags = reinterpret_cast<unsigned long long *>(b + o_lbflags);
    h->lb_ready = reinterpret_cast<unsigned int *>(b + o_lbready);
    *out = h;
    return EP_OK;
}

EP_API int ep_handle_destroy(ep_handle *h) {
    if (!h) return EP_ERR_ARG;
    int rc = EP_OK;
    {
        DeviceGuard g(h->device);
        if (g.err != cudaSuccess) rc = cuda_fail(g.err, "cudaSetDevice");
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess && rc == EP_OK) rc = cuda_fail(e, "cudaDeviceSynchronize");
        e = cudaFree(h->block);
        if (e != cudaSuccess && rc == EP_OK) rc = cuda_fail(e, "cudaFree(handle)");
    }
    delete h;
    return rc;
}

EP_API int ep_handle_get_view(const ep_handle *h, ep_handle_view *v) {
    if (!h || !v) return EP_ERR_ARG;
    v->pos = h->pos;
    v->row_src = h->row_src;
    v->row_slot = h->row_slot;
    v->row_weight = h->row_weight;
    v->num_tokens_per_expert = h->cnt;
    v->num_tokens_per_rank = h->rank_tok;
    v->expert_offsets = h->eoff;
    v->rank_offsets = h->roff;
    v->status = h->status;
    v->capacity = h->cap;
    return EP_OK;
}

EP_API int ep_get_layout(ep_handle *h, const int64_t *topk_idx, const float *topk_weights,
                         int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                         uint8_t *is_token_in_rank, int32_t *expert_offsets, int32_t *rank_offsets,
                         ep_stream_t stream) {
    int rc = check_mode(h, false, false);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (c.num_tokens > 0 && !topk_idx) return EP_ERR_ARG;
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(num_tokens_per_expert, 4) ||
        !aligned(num_tokens_per_rank, 4) || !aligned(expert_offsets, 4) || !aligned(rank_offsets, 4))
        return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");

    ep::LayoutParams p{};
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.T = c.num_tokens;
    p.K = c.num_topk;
    p.E = c.num_experts;
    p.R = c.num_ranks;
    p.L = c.num_experts / c.num_ranks;
    p.A = c.expert_alignment;
    p.id_bits = 0;
    while ((1 << p.id_bits) < c.num_experts) ++p.id_bits;
    p.G = h->G;
    p.G_stride = (h->G + 3) / 4 * 4;
    p.tokens_per_chunk = h->tokens_per_chunk;
    p.pos = h->pos;
    p.row_src = h->row_src;
    p.row_slot = h->row_slot;
    p.row_weight = h->row_weight;
    p.cnt = h->cnt;
    p.rank_tok = h->rank_tok;
    p.eoff = h->eoff;
    p.roff = h->roff;
    p.u_cnt = num_tokens_per_expert;
    p.u_rank_tok = num_tokens_per_rank;
    p.u_eoff = expert_offsets;
    p.u_roff = rank_offsets;
    p.u_in_rank = is_token_in_rank;
    p.chunk_counts = h->chunk_counts;
    p.barrier = h->barrier;
    p.status = h->status;
    p.wait_limit_ns = h->wait_limit_ns;
    p.barrier_extra = h->barrier_extra;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    cudaError_t e;
    if (c.num_tokens > 0 && c.num_tokens < 2 * sms) {
        // fewer than two tokens per SM: one CTA per token, each counting all
        // pairs itself (the small-batch kernel without its copy)
        ep::DispatchParams d{};
        d.H = c.hidden;
        d.T = c.num_tokens;
        d.K = c.num_topk;
        d.E = c.num_experts;
        d.status = h->status;
        e = ep::launch_layout_dispatch_small(d, p, false, sms, reinterpret_cast<cudaStream_t>(stream));
    } else {
        e = ep::launch_layout(p, h->plan, reinterpret_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "launch(layout)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    h->has_layout = true;
    return EP_OK;
}

static ep::LbParams lb_params(const ep_handle *h, const void *x, void *recv, float *scales, int lb);

static int dispatch_common(const ep_handle *h, const void *x, void *recv, float *scales, bool fp8,
                           ep_stream_t stream) {
    int rc = check_mode(h, false, true);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (fp8 && c.hidden % 128 != 0) return EP_ERR_ARG;
    if (c.num_tokens == 0) return EP_OK;   // nothing to write: rows == 0
    if (!x || !recv || (fp8 && !scales)) return EP_ERR_ARG;
    if (!aligned(x, 16) || !aligned(recv, 16) || !aligned(scales, 4)) return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");

    ep::DispatchParams p{};
    p.x = x;
    p.recv = recv;
    p.recv_scale = scales;
    p.scale_ld = h->scale_layout == EP_SCALES_COL_MAJOR_TMA ? (int)((h->cap + 3) / 4 * 4) : 0;
    p.scale_group_rows = (int)h->cap;
    p.pos = h->pos;
    p.row_src = h->row_src;
    p.eoff = h->eoff;
    p.T = c.num_tokens;
    p.K = c.num_topk;
    p.E = c.num_experts;
    p.H = c.hidden;
    p.status = h->status;
    p.wait_limit_ns = h->wait_limit_ns;
    p.splits = 1;
    p.n_token_units = p.T * p.splits;
    p.n_zero_units = c.expert_alignment > 1
                         ? (int)((h->cap + ep::kZeroRowsPerUnit - 1) / ep::kZeroRowsPerUnit)
                         : 0;
    // x is pulled into L2 ahead of the gather only when it fits in half of it:
    // a larger x pinned with evict_last would push out its own rows before use
    p.prefetch_x = (int64_t)c.num_tokens * c.hidden * 2 <= (int64_t)h->l2_bytes / 2;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    // Batches that fill the GPU (at least two tokens per SM) take the chunked
    // kernel of dispatch_lb.cu with its dynamically claimed copy order (against
    // the earlier staged bf16 / register FP8 kernels: dsv3 bf16 93.6 -> 90.8 us,
    // large FP8 260.2 -> 218.2 us in one A/B run); smaller ones the register
    // kernels of dispatch.cu.
    const bool chunked = c.num_tokens >= 2 * sms && c.num_tokens < ep::kLbMaxTokens;
    cudaError_t e = chunked ? ep::launch_dispatch_lb(lb_params(h, x, recv, scales, 0), fp8, sms, s)
                    : fp8   ? ep::launch_dispatch_fp8(p, sms, s)
                            : ep::launch_dispatch_bf16(p, sms, s);
    if (e != cudaSuccess) return cuda_fail(e, fp8 ? "launch(dispatch_fp8)" : "launch(dispatch)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return EP_OK;
}

EP_API int ep_dispatch(const ep_handle *h, const void *x, void *recv_x, ep_stream_t stream) {
    return dispatch_common(h, x, recv_x, nullptr, false, stream);
}

EP_API int ep_dispatch_fp8(const ep_handle *h, const void *x, void *recv_q, float *recv_scales,
                           ep_stream_t stream) {
    return dispatch_common(h, x, recv_q, recv_scales, true, stream);
}

// The handle's arrays and the fused path's scratch, for the chunked dispatch
// kernel (lb = 1: layout in the kernel; lb = 0: positions from the handle).
static ep::LbParams lb_params(const ep_handle *h, const void *x, void *recv, float *scales, int lb) {
    const ep_config &c = h->cfg;
    ep::LbParams p{};
    p.x = x;
    p.recv = recv;
    p.recv_scale = scales;
    p.scale_ld = h->scale_layout == EP_SCALES_COL_MAJOR_TMA ? (int)((h->cap + 3) / 4 * 4) : 0;
    p.pos = h->pos;
    p.row_src = h->row_src;
    p.row_slot = h->row_slot;
    p.row_weight = h->row_weight;
    p.cnt = h->cnt;
    p.rank_tok = h->rank_tok;
    p.eoff = h->eoff;
    p.roff = h->roff;
    p.super_hist = h->lb_super_hist;
    p.super_base = h->lb_super_base;
    p.flags = h->lb_flags;
    p.ready = h->lb_ready;
    p.ctl = h->lb_ctl;
    p.status = h->status;
    p.wait_limit_ns = h->wait_limit_ns;
    p.stall_first_chunk = lb && h->barrier_extra > 0;
    p.T = c.num_tokens;
    p.K = c.num_topk;
    p.E = c.num_experts;
    p.R = c.num_ranks;
    p.L = c.num_experts / c.num_ranks;
    p.A = c.expert_alignment;
    p.H = c.hidden;
    p.id_bits = 0;
    while ((1 << p.id_bits) < c.num_experts) ++p.id_bits;
    p.nchunks = h->lb.nchunks;
    p.tpc = h->lb.tpc;
    p.nsuper = h->lb.nsuper;
    p.lb = lb;
    p.prefetch_x = (int64_t)c.num_tokens * c.hidden * 2 <= (int64_t)h->l2_bytes / 2;
    return p;
}

static int layout_dispatch_common(ep_handle *h, const int64_t *topk_idx, const float *topk_weights, const void *x,
                                  void *recv, float *scales, bool fp8, int32_t *num_tokens_per_expert,
                                  int32_t *num_tokens_per_rank, uint8_t *is_token_in_rank, int32_t *expert_offsets,
                                  int32_t *rank_offsets, ep_stream_t stream) {
    int rc = check_mode(h, false, false);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (fp8 && c.hidden % 128 != 0) return EP_ERR_ARG;
    if (c.num_tokens >= ep::kLbMaxTokens) {
        ep::record_error("ep_layout_dispatch: at most 2^22 - 1 tokens per call");
        return EP_ERR_UNSUPPORTED;
    }
    if (c.num_tokens > 0 && (!topk_idx || !x || !recv || (fp8 && !scales))) return EP_ERR_ARG;
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(x, 16) || !aligned(recv, 16) ||
        !aligned(scales, 4) || !aligned(num_tokens_per_expert, 4) || !aligned(num_tokens_per_rank, 4) ||
        !aligned(expert_offsets, 4) || !aligned(rank_offsets, 4))
        return EP_ERR_ARG;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    if (c.num_tokens > 0 && c.num_tokens < 2 * sms) {
        // too few tokens to fill the GPU: one launch, one CTA per token, each
        // counting all pairs itself (decode: 17.9 us for the layout kernel and
        // the register dispatch, 31.6 us for the chunked kernel with look-back)
        ep::LayoutParams lp{};
        lp.topk_idx = topk_idx;
        lp.topk_weights = topk_weights;
        lp.T = c.num_tokens;
        lp.K = c.num_topk;
        lp.E = c.num_experts;
        lp.R = c.num_ranks;
        lp.L = c.num_experts / c.num_ranks;
        lp.A = c.expert_alignment;
        lp.pos = h->pos;
        lp.row_src = h->row_src;
        lp.row_slot = h->row_slot;
        lp.row_weight = h->row_weight;
        lp.cnt = h->cnt;
        lp.rank_tok = h->rank_tok;
        lp.eoff = h->eoff;
        lp.roff = h->roff;
        lp.u_cnt = num_tokens_per_expert;
        lp.u_rank_tok = num_tokens_per_rank;
        lp.u_eoff = expert_offsets;
        lp.u_roff = rank_offsets;
        lp.u_in_rank = is_token_in_rank;
        lp.status = h->status;
        lp.wait_limit_ns = h->wait_limit_ns;
        ep::DispatchParams p{};
        p.x = x;
        p.recv = recv;
        p.recv_scale = scales;
        p.scale_ld = h->scale_layout == EP_SCALES_COL_MAJOR_TMA ? (int)((h->cap + 3) / 4 * 4) : 0;
        p.scale_group_rows = (int)h->cap;
        p.H = c.hidden;
        p.T = c.num_tokens;
        p.K = c.num_topk;
        p.E = c.num_experts;
        p.status = h->status;
        cudaError_t e = ep::launch_layout_dispatch_small(p, lp, fp8, sms, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, fp8 ? "launch(layout_dispatch_fp8)" : "launch(layout_dispatch)");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        h->has_layout = true;
        return EP_OK;
    }
    ep::LbParams p = lb_params(h, x, recv, scales, 1);
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.u_cnt = num_tokens_per_expert;
    p.u_rank_tok = num_tokens_per_rank;
    p.u_in_rank = is_token_in_rank;
    p.u_eoff = expert_offsets;
    p.u_roff = rank_offsets;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = ep::launch_layout_counts(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "launch(layout_counts)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    h->has_layout = true;
    if (c.num_tokens == 0) return EP_OK;
    e = ep::launch_dispatch_lb(p, fp8, sms, s);
    if (e != cudaSuccess) return cuda_fail(e, fp8 ? "launch(layout_dispatch_fp8)" : "launch(layout_dispatch)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return EP_OK;
}

EP_API int ep_layout_dispatch(ep_handle *h, const int64_t *topk_idx, const float *topk_weights, const void *x,
                              void *recv_x, int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                              uint8_t *is_token_in_rank, int32_t *expert_offsets, int32_t *rank_offsets,
                              ep_stream_t stream) {
    return layout_dispatch_common(h, topk_idx, topk_weights, x, recv_x, nullptr, false, num_tokens_per_expert,
                                  num_tokens_per_rank, is_token_in_rank, expert_offsets, rank_offsets, stream);
}

EP_API int ep_layout_dispatch_fp8(ep_handle *h, const int64_t *topk_idx, const float *topk_weights, const void *x,
                                  void *recv_q, float *recv_scales, int32_t *num_tokens_per_expert,
                                  int32_t *num_tokens_per_rank, uint8_t *is_token_in_rank, int32_t *expert_offsets,
                                  int32_t *rank_offsets, ep_stream_t stream) {
    return layout_dispatch_common(h, topk_idx, topk_weights, x, recv_q, recv_scales, true, num_tokens_per_expert,
                                  num_tokens_per_rank, is_token_in_rank, expert_offsets, rank_offsets, stream);
}

static int combine_common(const ep_handle *h, const void *y, const float *topk_weights, void *out,
                          bool ll, ep_stream_t stream) {
    int rc = check_mode(h, ll, true);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (c.num_tokens == 0) return EP_OK;
    if (!y || !topk_weights || !out) return EP_ERR_ARG;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(topk_weights, 4)) return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");

    ep::CombineParams p{};
    p.y = y;
    p.w = topk_weights;
    p.out = out;
    p.pos = h->pos;
    p.T = c.num_tokens;
    p.K = c.num_topk;
    p.H = c.hidden;
    p.status = h->status;
    p.wait_limit_ns = h->wait_limit_ns;
    p.splits = 1;
    p.n_units = p.T * p.splits;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    cudaError_t e = ep::launch_combine(p, sms, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launch(combine)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return EP_OK;
}

EP_API int ep_combine(const ep_handle *h, const void *y, const float *topk_weights, void *out,
                      ep_stream_t stream) {
    return combine_common(h, y, topk_weights, out, false, stream);
}

EP_API int ep_ll_combine(const ep_handle *h, const void *y, const float *topk_weights, void *out,
                         ep_stream_t stream) {
    return combine_common(h, y, topk_weights, out, true, stream);
}

static int expert_combine_common(const ep_handle *h, const void *act, const float *act_scales, int32_t inner,
                                 const void *w, const float *w_scales, int32_t n_out, const float *topk_weights,
                                 float *out_acc, void *out, bool fp8, ep_stream_t stream) {
    int rc = check_mode(h, false, true);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (c.expert_alignment % 128 != 0 || inner <= 0 || inner % (fp8 ? 128 : 64) != 0 || n_out <= 0 ||
        n_out % 256 != 0)
        return EP_ERR_ARG;
    if ((int64_t)c.num_experts * n_out > INT32_MAX || h->cap > INT32_MAX) return EP_ERR_UNSUPPORTED;
    if (c.num_tokens == 0) return EP_OK;
    if (!act || !w || !topk_weights || !out_acc || !out) return EP_ERR_ARG;
    if (fp8 && (!act_scales || !w_scales || !aligned(act_scales, 4) || !aligned(w_scales, 4))) return EP_ERR_ARG;
    if (!aligned(act, 16) || !aligned(w, 16) || !aligned(out_acc, 16) || !aligned(out, 16) ||
        !aligned(topk_weights, 4))
        return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    ep::GemmCombineArgs a{};
    a.p.eoff = h->eoff;
    a.p.row_src = h->row_src;
    a.p.row_slot = h->row_slot;
    a.p.topk_w = topk_weights;
    a.p.out_acc = out_acc;
    a.p.status = h->status;
    a.p.wait_limit_ns = h->wait_limit_ns;
    a.p.E = c.num_experts;
    a.p.K = c.num_topk;
    a.p.N = n_out;
    a.p.I = inner;
    a.p.act_scale = act_scales;
    a.p.w_scale = w_scales;
    a.p.scale_ld = h->scale_layout == EP_SCALES_COL_MAJOR_TMA ? (int)((h->cap + 3) / 4 * 4) : 0;
    a.fp8 = fp8;
    a.act = act;
    a.w = w;
    a.out = out;
    a.cap = h->cap;
    a.T = c.num_tokens;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    cudaError_t e = ep::launch_gemm_combine(a, sms, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, fp8 ? "launch(expert_combine_fp8)" : "launch(expert_combine)");
    g_launches.fetch_add(2, std::memory_order_relaxed);
    return EP_OK;
}

EP_API int ep_expert_combine(const ep_handle *h, const void *act, int32_t inner, const void *w, int32_t n_out,
                             const float *topk_weights, float *out_acc, void *out, ep_stream_t stream) {
    return expert_combine_common(h, act, nullptr, inner, w, nullptr, n_out, topk_weights, out_acc, out, false,
                                 stream);
}

EP_API int ep_expert_combine_fp8(const ep_handle *h, const uint8_t *act_q, const float *act_scales, int32_t inner,
                                 const uint8_t *w_q, const float *w_scales, int32_t n_out,
                                 const float *topk_weights, float *out_acc, void *out, ep_stream_t stream) {
    return expert_combine_common(h, act_q, act_scales, inner, w_q, w_scales, n_out, topk_weights, out_acc, out,
                                 true, stream);
}

// ---- peer-memory exchange (one process per GPU) ----

enum class PeerOp { kDispatch, kDispatchFp8, kCombine };

static int peer_common(const ep_handle *h, PeerOp op, const void *x, const void *const *bases,
                       float *const *scale_bases, const int32_t *row0, const float *topk_weights, void *out,
                       ep_stream_t stream) {
    int rc = check_mode(h, false, true);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (op == PeerOp::kDispatchFp8 && (c.hidden % 128 != 0 || !scale_bases || !aligned(scale_bases, 8)))
        return EP_ERR_ARG;
    if (op == PeerOp::kDispatchFp8 && h->scale_layout != EP_SCALES_ROW_MAJOR) return EP_ERR_UNSUPPORTED;
    if (c.num_tokens == 0) return EP_OK;
    if (!bases || !row0 || !aligned(bases, 8) || !aligned(row0, 4)) return EP_ERR_ARG;
    if (op == PeerOp::kCombine ? (!topk_weights || !out || !aligned(topk_weights, 4) || !aligned(out, 16))
                               : (!x || !aligned(x, 16)))
        return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");

    ep::PeerLaunch l{};
    l.x = x;
    l.base = const_cast<void *const *>(bases);
    l.sbase = scale_bases;
    l.row0 = row0;
    l.pos = h->pos;
    l.row_src = h->row_src;
    l.roff = h->roff;
    l.w = topk_weights;
    l.out = out;
    l.T = c.num_tokens;
    l.K = c.num_topk;
    l.R = c.num_ranks;
    l.H = c.hidden;
    l.cap = h->cap;
    l.zero_rows = c.expert_alignment > 1;
    l.prefetch_x = (int64_t)c.num_tokens * c.hidden * 2 <= (int64_t)h->l2_bytes / 2;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    const char *what;
    switch (op) {
        case PeerOp::kDispatch: e = ep::launch_dispatch_peer(l, sms, s); what = "launch(dispatch_peer)"; break;
        case PeerOp::kDispatchFp8:
            e = ep::launch_dispatch_fp8_peer(l, sms, s);
            what = "launch(dispatch_fp8_peer)";
            break;
        default: e = ep::launch_combine_peer(l, sms, s); what = "launch(combine_peer)"; break;
    }
    if (e != cudaSuccess) return cuda_fail(e, what);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return EP_OK;
}

EP_API int ep_dispatch_peer(const ep_handle *h, const void *x, void *const *recv_bases, const int32_t *row0,
                            ep_stream_t stream) {
    return peer_common(h, PeerOp::kDispatch, x, const_cast<const void *const *>(recv_bases), nullptr, row0,
                       nullptr, nullptr, stream);
}

EP_API int ep_dispatch_peer_fp8(const ep_handle *h, const void *x, void *const *recv_bases,
                                float *const *scale_bases, const int32_t *row0, ep_stream_t stream) {
    return peer_common(h, PeerOp::kDispatchFp8, x, const_cast<const void *const *>(recv_bases), scale_bases, row0,
                       nullptr, nullptr, stream);
}

EP_API int ep_combine_peer(const ep_handle *h, const void *const *y_bases, const int32_t *row0,
                           const float *topk_weights, void *out, ep_stream_t stream) {
    return peer_common(h, PeerOp::kCombine, nullptr, y_bases, nullptr, row0, topk_weights, out, stream);
}

static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");

// cuMemGetAddressRange through the runtime's driver entry point (no libcuda link).
typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

static AddressRangeFn address_range_fn() {
    static AddressRangeFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(f);
    }
    return fn;
}

EP_API int ep_ipc_get_handle(const void *dev_ptr, void *handle, int64_t *offset) {
    if (!dev_ptr || !handle || !offset) return EP_ERR_ARG;
    AddressRangeFn range = address_range_fn();
    if (!range) {
        ep::record_error("cuMemGetAddressRange entry point unavailable");
        return EP_ERR_UNSUPPORTED;
    }
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return EP_ERR_ARG;
    cudaIpcMemHandle_t hd;
    cudaError_t e = cudaIpcGetMemHandle(&hd, reinterpret_cast<void *>(base));
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
    memcpy(handle, &hd, sizeof hd);
    *offset = static_cast<int64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
    return EP_OK;
}

EP_API int ep_ipc_open_handle(const void *handle, void **base) {
    if (!handle || !base) return EP_ERR_ARG;
    cudaIpcMemHandle_t hd;
    memcpy(&hd, handle, sizeof hd);
    cudaError_t e = cudaIpcOpenMemHandle(base, hd, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
    return EP_OK;
}

EP_API int ep_ipc_close_handle(void *base) {
    if (!base) return EP_ERR_ARG;
    cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
    return EP_OK;
}

// ---- low-latency (static, masked) layout ----

EP_API int64_t ep_ll_capacity_rows(const ep_config *c, int32_t M) {
    int rc = ep_validate_config(c);
    if (rc != EP_OK) return rc;
    if (M < 1 || M < c->num_tokens) return EP_ERR_ARG;
    const int64_t cap = (int64_t)c->num_experts * M;
    if (cap > INT32_MAX) return EP_ERR_UNSUPPORTED;
    return cap;
}

EP_API int64_t ep_ll_scale_buffer_floats(const ep_config *c, int32_t M, int32_t layout) {
    const int64_t cap = ep_ll_capacity_rows(c, M);
    if (cap < 0) return cap;
    if (c->hidden % 128 != 0) return EP_ERR_ARG;
    const int64_t nb = c->hidden / 128;
    if (layout == EP_SCALES_ROW_MAJOR) return cap * nb;
    if (layout == EP_SCALES_COL_MAJOR_TMA) return (int64_t)c->num_experts * nb * ((M + 3) / 4 * 4);
    return EP_ERR_ARG;
}

EP_API int ep_ll_handle_create(const ep_config *cfg, int32_t M, ep_handle **out) {
    if (!out) return EP_ERR_ARG;
    *out = nullptr;
    const int64_t cap = ep_ll_capacity_rows(cfg, M);
    if (cap < 0) return (int)cap;
    ep_handle *h = new (std::nothrow) ep_handle();
    if (!h) return EP_ERR_ARG;
    h->cfg = *cfg;
    h->cap = cap;
    h->ll_M = M;
    h->wait_limit_ns = ep::kDefaultWaitLimitNs;
    h->scale_layout = EP_SCALES_ROW_MAJOR;
    auto fail = [&](int code) {
        delete h;
        return code;
    };
    cudaError_t e = cudaGetDevice(&h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaGetDevice"));
    e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaDeviceGetAttribute"));
    const size_t o_stat = round_up(sizeof(int32_t) * (size_t)cfg->num_tokens * cfg->num_topk + 1, 256);
    const size_t o_bar = o_stat + 256;
    h->block_bytes = o_bar + round_up(sizeof(ep::GridBarrier), 256);
    e = cudaMalloc(&h->block, h->block_bytes);
    if (e != cudaSuccess) return fail(cuda_fail(e, "cudaMalloc(handle)"));
    e = cudaMemset(h->block, 0, h->block_bytes);
    if (e != cudaSuccess) {
        cudaFree(h->block);
        return fail(cuda_fail(e, "cudaMemset(handle)"));
    }
    char *b = static_cast<char *>(h->block);
    h->pos = reinterpret_cast<int32_t *>(b);
    h->status = reinterpret_cast<unsigned int *>(b + o_stat);
    h->barrier = reinterpret_cast<ep::GridBarrier *>(b + o_bar);
    *out = h;
    return EP_OK;
}

static int ll_dispatch_common(ep_handle *h, const int64_t *topk_idx, const void *x, void *recv,
                              float *scales, int32_t *recv_count, bool fp8, ep_stream_t stream) {
    int rc = check_mode(h, true, false);
    if (rc != EP_OK) return rc;
    const ep_config &c = h->cfg;
    if (fp8 && c.hidden % 128 != 0) return EP_ERR_ARG;
    if (!aligned(recv_count, 4)) return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (c.num_tokens == 0) {   // no pairs: every expert's count is 0
        if (recv_count) EP_CUDA(cudaMemsetAsync(recv_count, 0, sizeof(int32_t) * c.num_experts, s));
        h->has_layout = true;
        return EP_OK;
    }
    if (!topk_idx || !x || !recv || (fp8 && !scales)) return EP_ERR_ARG;
    if (!aligned(topk_idx, 8) || !aligned(x, 16) || !aligned(recv, 16) || !aligned(scales, 4))
        return EP_ERR_ARG;

    ep::DispatchParams p{};
    p.x = x;
    p.recv = recv;
    p.recv_scale = scales;
    p.scale_ld = h->scale_layout == EP_SCALES_COL_MAJOR_TMA ? (h->ll_M + 3) / 4 * 4 : 0;
    p.scale_group_rows = h->ll_M;
    p.T = c.num_tokens;
    p.K = c.num_topk;
    p.E = c.num_experts;
    p.H = c.hidden;
    p.status = h->status;
    p.wait_limit_ns = h->wait_limit_ns;
    p.ll_M = h->ll_M;
    p.topk_idx = topk_idx;
    p.pos_out = h->pos;
    p.recv_count = recv_count;
    const int sms = h->sm_limit > 0 && h->sm_limit < h->num_sms ? h->sm_limit : h->num_sms;
    cudaError_t e = ep::launch_ll_dispatch(p, fp8, sms, s);
    if (e != cudaSuccess) return cuda_fail(e, fp8 ? "launch(ll_dispatch_fp8)" : "launch(ll_dispatch)");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    h->has_layout = true;
    return EP_OK;
}

EP_API int ep_ll_dispatch(ep_handle *h, const int64_t *topk_idx, const void *x, void *recv_x,
                          int32_t *recv_count, ep_stream_t stream) {
    return ll_dispatch_common(h, topk_idx, x, recv_x, nullptr, recv_count, false, stream);
}

EP_API int ep_ll_dispatch_fp8(ep_handle *h, const int64_t *topk_idx, const void *x, void *recv_q,
                              float *recv_scales, int32_t *recv_count, ep_stream_t stream) {
    return ll_dispatch_common(h, topk_idx, x, recv_q, recv_scales, recv_count, true, stream);
}

EP_API int ep_copy_routing(const ep_handle *h, int32_t *pos, int32_t *row_src, int32_t *row_slot,
                           float *row_weight, ep_stream_t stream) {
    int rc = check_handle(h, true);
    if (rc != EP_OK) return rc;
    if (!aligned(pos, 4) || !aligned(row_src, 4) || !aligned(row_slot, 4) || !aligned(row_weight, 4))
        return EP_ERR_ARG;
    if (h->ll_M > 0 && (row_src || row_slot || row_weight)) return EP_ERR_ARG;   // pos only
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t npairs = (size_t)h->cfg.num_tokens * h->cfg.num_topk, ncap = (size_t)h->cap;
    const cudaMemcpyKind d2d = cudaMemcpyDeviceToDevice;
    if (pos && npairs) EP_CUDA(cudaMemcpyAsync(pos, h->pos, sizeof(int32_t) * npairs, d2d, s));
    if (row_src && ncap) EP_CUDA(cudaMemcpyAsync(row_src, h->row_src, sizeof(int32_t) * ncap, d2d, s));
    if (row_slot && ncap) EP_CUDA(cudaMemcpyAsync(row_slot, h->row_slot, sizeof(int32_t) * ncap, d2d, s));
    if (row_weight && ncap) EP_CUDA(cudaMemcpyAsync(row_weight, h->row_weight, sizeof(float) * ncap, d2d, s));
    return EP_OK;
}

EP_API int ep_get_num_rows(const ep_handle *h, int32_t *rows, ep_stream_t stream) {
    int rc = check_mode(h, false, true);
    if (rc != EP_OK) return rc;
    if (!rows) return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    EP_CUDA(cudaMemcpyAsync(rows, h->eoff + h->cfg.num_experts, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    EP_CUDA(cudaStreamSynchronize(s));
    return EP_OK;
}

EP_API int ep_get_status(const ep_handle *h, uint32_t *bits, ep_stream_t stream) {
    int rc = check_handle(h, false);
    if (rc != EP_OK) return rc;
    if (!bits) return EP_ERR_ARG;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    EP_CUDA(cudaMemcpyAsync(bits, h->status, sizeof(uint32_t), cudaMemcpyDeviceToHost, s));
    EP_CUDA(cudaStreamSynchronize(s));
    return *bits ? EP_ERR_DEVICE : EP_OK;
}

EP_API int ep_clear_status(ep_handle *h, ep_stream_t stream) {
    int rc = check_handle(h, false);
    if (rc != EP_OK) return rc;
    DeviceGuard g(h->device);
    if (g.err != cudaSuccess) return cuda_fail(g.err, "cudaSetDevice");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    EP_CUDA(cudaMemsetAsync(h->status, 0, sizeof(unsigned int), s));
    EP_CUDA(cudaMemsetAsync(h->barrier, 0, sizeof(ep::GridBarrier), s));
    if (h->lb_ctl)   // arrival counters and tickets; the epoch stays, so earlier look-back words never match
        EP_CUDA(cudaMemsetAsync(h->lb_ctl, 0, offsetof(ep::LbControl, epoch), s));
    return EP_OK;
}

EP_API int ep_set_scale_layout(ep_handle *h, int32_t layout) {
    if (!h || (layout != EP_SCALES_ROW_MAJOR && layout != EP_SCALES_COL_MAJOR_TMA)) return EP_ERR_ARG;
    h->scale_layout = layout;
    return EP_OK;
}

EP_API int ep_set_sm_limit(ep_handle *h, int32_t num_sms) {
    if (!h || num_sms < 0) return EP_ERR_ARG;
    h->sm_limit = num_sms;
    return EP_OK;
}

EP_API int ep_set_wait_limit(ep_handle *h, uint64_t limit_ns, int32_t extra_arrivals) {
    if (!h || limit_ns == 0 || extra_arrivals < 0) return EP_ERR_ARG;
    h->wait_limit_ns = limit_ns;
    h->barrier_extra = extra_arrivals;
    return EP_OK;
}

EP_API const char *ep_status_string(int code) {
    switch (code) {
        case EP_OK: return "ok";
        case EP_ERR_ARG: return "invalid argument (null pointer, size, alignment or E % R != 0)";
        case EP_ERR_CUDA: return "CUDA runtime error (see ep_last_error)";
        case EP_ERR_UNSUPPORTED: return "sizes beyond the library's limits";
        case EP_ERR_STATE: return "handle has no layout yet, or is of the other layout mode";
        case EP_ERR_DEVICE: return "device reported an error (bad expert id, wait timeout or slot overflow)";
        default: return "unknown status";
    }
}

EP_API const char *ep_last_error(void) { return g_last_error; }

EP_API uint64_t ep_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
