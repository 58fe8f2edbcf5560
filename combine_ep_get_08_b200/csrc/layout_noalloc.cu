// layout_noalloc.cu -- the layout without any device allocation.
//
// ep_get_layout needs a handle, and ep_handle_create calls cudaMalloc.
// Some callers cannot do that at the point where they route tokens: code
// that must not trigger a device allocation (which can synchronise the
// device or fail under memory pressure), runtimes that hand out device
// memory only from their own pools, or code that otherwise has no place to
// keep a handle.  For them this file offers one entry point that takes every
// output from the caller and keeps the kernel's scratch (the per-chunk
// expert histograms and the grid-wide arrival counter) in a fixed
// file-scope device array, which each GPU that loads the library holds until
// the process exits.
#include <cstdio>
#include <mutex>

#include "ep_internal.cuh"

namespace {

// 256 KiB: the arrival counter in the first 256 bytes, then the chunk
// histograms, (E + R) rows of G rounded up to 4 int32 each.
constexpr size_t kScratchBytes = 256 * 1024;
constexpr size_t kCountsOffset = 256;

static __device__ __align__(256) unsigned char g_layout_scratch[kScratchBytes];

using ep::kMaxDevices;

struct DeviceSetup {
    bool ready;
    unsigned char *scratch;   // device address of g_layout_scratch on this device
    int num_sms;
};

std::mutex g_setup_mutex;
DeviceSetup g_setup[kMaxDevices];

// Once per device, with that device current: resolve the array's device
// address (in host code its name only stands for it), allow the layout
// kernel's dynamic shared memory, and read the SM count.
int setup_device(int dev, DeviceSetup *out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    DeviceSetup &s = g_setup[dev];
    if (!s.ready) {
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_layout_scratch);
        if (e != cudaSuccess) return ep::record_cuda_error(e, "cudaGetSymbolAddress(layout scratch)");
        e = ep::layout_prepare(dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return ep::record_cuda_error(e, "layout set-up");
        s.scratch = static_cast<unsigned char *>(ptr);
        s.ready = true;
    }
    *out = s;
    return EP_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Bytes of the array a layout of this launch shape uses: none for the
// cluster kernel; the arrival counter and the chunk histograms (E + R rows of
// G rounded up to 4 int32) for the cooperative kernel.
size_t scratch_need(const ep::LayoutPlan &plan, int E, int R) {
    if (plan.cluster) return 0;
    const size_t G_stride = ((size_t)plan.G + 3) / 4 * 4;
    return kCountsOffset + sizeof(int32_t) * G_stride * (size_t)(E + R);
}

// The current device, checked against the table size.
int current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return ep::record_cuda_error(e, "cudaGetDevice");
    if (*dev < 0 || *dev >= kMaxDevices) {
        ep::record_error("device ordinal beyond the 64 this library tracks");
        return EP_ERR_UNSUPPORTED;
    }
    return EP_OK;
}

}  // namespace

extern "C" {

EP_API int ep_get_layout_noalloc(const ep_config *cfg, const int64_t *topk_idx, const float *topk_weights,
                                 int32_t *pos, int32_t *row_src, int32_t *row_slot, float *row_weight,
                                 int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                                 uint8_t *is_token_in_rank, int32_t *expert_offsets, int32_t *rank_offsets,
                                 uint32_t *status, ep_stream_t stream) {
    int rc = ep_validate_config(cfg);
    if (rc != EP_OK) return rc;
    const int T = cfg->num_tokens, E = cfg->num_experts, R = cfg->num_ranks, K = cfg->num_topk;
    if ((T > 0 && !topk_idx) || !pos || !row_src || !row_slot || (topk_weights && !row_weight) ||
        !num_tokens_per_expert || !num_tokens_per_rank || !expert_offsets || !rank_offsets || !status)
        return EP_ERR_ARG;
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(pos, 4) || !aligned(row_src, 4) ||
        !aligned(row_slot, 4) || !aligned(row_weight, 4) || !aligned(num_tokens_per_expert, 4) ||
        !aligned(num_tokens_per_rank, 4) || !aligned(expert_offsets, 4) || !aligned(rank_offsets, 4) ||
        !aligned(status, 4))
        return EP_ERR_ARG;

    int dev = 0;
    rc = current_device(&dev);
    if (rc != EP_OK) return rc;
    DeviceSetup s;
    rc = setup_device(dev, &s);
    if (rc != EP_OK) return rc;

    // same launch shape as a handle's layout; only the cooperative fallback
    // uses the scratch array
    const ep::LayoutPlan plan = ep::plan_layout(dev, T, E, R, K, s.num_sms);
    const int64_t G = plan.G;
    const int tpc = plan.tokens_per_chunk;
    const int G_stride = (int)((G + 3) / 4 * 4);
    const size_t need = scratch_need(plan, E, R);
    if (need > kScratchBytes) {
        char msg[160];
        snprintf(msg, sizeof msg, "ep_get_layout_noalloc: %zu bytes of scratch needed, the fixed array holds %zu",
                 need, kScratchBytes);
        ep::record_error(msg);
        return EP_ERR_UNSUPPORTED;
    }

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the arrival counter and
    // the histogram rows (whose tail past G is read as zeros) start at zero
    cudaError_t e = need ? cudaMemsetAsync(s.scratch, 0, need, st) : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return ep::record_cuda_error(e, "cudaMemsetAsync(layout scratch)");

    ep::LayoutParams p{};
    p.topk_idx = topk_idx;
    p.topk_weights = topk_weights;
    p.T = T;
    p.K = K;
    p.E = E;
    p.R = R;
    p.L = E / R;
    p.A = cfg->expert_alignment;
    p.id_bits = 0;
    while ((1 << p.id_bits) < E) ++p.id_bits;
    p.G = (int)G;
    p.G_stride = G_stride;
    p.tokens_per_chunk = tpc;
    p.pos = pos;
    p.row_src = row_src;
    p.row_slot = row_slot;
    p.row_weight = row_weight;
    p.cnt = num_tokens_per_expert;
    p.rank_tok = num_tokens_per_rank;
    p.eoff = expert_offsets;
    p.roff = rank_offsets;
    p.u_in_rank = is_token_in_rank;
    p.chunk_counts = reinterpret_cast<int32_t *>(s.scratch + kCountsOffset);
    p.barrier = reinterpret_cast<ep::GridBarrier *>(s.scratch);
    p.status = status;
    p.wait_limit_ns = ep::kDefaultWaitLimitNs;
    p.barrier_extra = 0;
    e = ep::launch_layout(p, plan, st);
    if (e != cudaSuccess) return ep::record_cuda_error(e, "launch(layout)");
    ep::count_launch();
    return EP_OK;
}

EP_API int ep_layout_shape(const ep_config *cfg, int32_t *cluster, int32_t *ctas, int64_t *noalloc_scratch_bytes) {
    int rc = ep_validate_config(cfg);
    if (rc != EP_OK) return rc;
    int dev = 0;
    rc = current_device(&dev);
    if (rc != EP_OK) return rc;
    DeviceSetup s;
    rc = setup_device(dev, &s);
    if (rc != EP_OK) return rc;
    const ep::LayoutPlan plan =
        ep::plan_layout(dev, cfg->num_tokens, cfg->num_experts, cfg->num_ranks, cfg->num_topk, s.num_sms);
    if (cluster) *cluster = plan.cluster ? 1 : 0;
    if (ctas) *ctas = plan.G;
    if (noalloc_scratch_bytes) *noalloc_scratch_bytes = (int64_t)scratch_need(plan, cfg->num_experts, cfg->num_ranks);
    return EP_OK;
}

}  // extern "C"
