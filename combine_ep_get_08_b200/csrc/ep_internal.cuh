// ep_internal.cuh -- shared definitions of the sm_100a dispatch/combine library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ep.h"

namespace ep {

// ---------------------------------------------------------------------------
// Limits and launch shapes
// ---------------------------------------------------------------------------
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopk = 64;
constexpr int kLayoutThreads = 1024;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kLayoutPairsPerCta = 1024;   // target (token, k) pairs per layout CTA
constexpr int kZeroRowsPerUnit = 8;    // padding rows zero-filled per work unit
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;

struct GridBarrier {
    unsigned int count;          // arrivals so far (grows by G per layout launch)
    unsigned int epoch;          // completed grid-wide waits: advanced on the device, so a
                                 // launch replayed from a CUDA graph finds its own target
};

// ---------------------------------------------------------------------------
// Kernel parameter blocks
// ---------------------------------------------------------------------------
struct LayoutParams {
    const int64_t *topk_idx;
    const float *topk_weights;   // may be null
    int T, K, E, R, L, A;
    int id_bits;                 // bits needed for an expert id: ceil(log2(E))
    int G;                       // CTAs == chunks
    int G_stride;                // row stride of chunk_counts: G rounded up to 4
    int tokens_per_chunk;
    // handle arrays
    int32_t *pos, *row_src, *row_slot;
    float *row_weight;
    int32_t *cnt, *rank_tok, *eoff, *roff;
    // caller copies (may be null)
    int32_t *u_cnt, *u_rank_tok, *u_eoff, *u_roff;
    uint8_t *u_in_rank;
    // scratch
    int32_t *chunk_counts;       // [E+R][G_stride] (one row per expert / rank column)
    GridBarrier *barrier;
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int barrier_extra;
};

struct DispatchParams {
    const void *x;               // [T, H] bf16
    void *recv;                  // [cap, H] bf16 or e4m3
    float *recv_scale;           // FP8 only: [cap, H/128], or [H/128][scale_ld] when scale_ld > 0
    int scale_ld;                // 0: row-major scales; > 0: column-major leading dimension
    const int32_t *pos;          // [T, K]
    const int32_t *row_src;      // [cap]
    const int32_t *eoff;         // [E+1]
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int T, K, E, H;
    int splits;                  // column splits per token
    int n_token_units;           // T * splits
    int n_zero_units;            // ceil(cap / kZeroRowsPerUnit) when A > 1, else 0
    int scale_group_rows;        // column-major scales: rows per [H/128][scale_ld] group
    int prefetch_x;              // 1: each CTA prefetches its x rows into L2 before the dependency wait
    // low-latency static layout (ll_M > 0): destinations computed in-kernel
    // from topk_idx, e*ll_M + slot; no padding rows, no zero fill
    int ll_M;                    // fixed slots per expert
    const int64_t *topk_idx;     // [T, K]
    int32_t *pos_out;            // [T, K] destination of every pair (-1: none)
    int32_t *recv_count;         // [E] slots used per expert (NULL: not written)
};

struct CombineParams {
    const void *y;               // [cap, H] bf16
    const float *w;              // [T, K]
    void *out;                   // [T, H] bf16
    const int32_t *pos;          // [T, K]
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int T, K, H;
    int splits;
    int n_units;
};

// Expert GEMM with the combine fused into its epilogue.
struct GemmCombineParams {
    const int32_t *eoff;         // [E+1] padded expert offsets (row block -> expert)
    const int32_t *row_src;      // [cap] token of a received row, -1 for padding
    const int32_t *row_slot;     // [cap] k of a received row
    const float *topk_w;         // [T, K]
    float *out_acc;              // [T, N] fp32 accumulator (zeroed by the launcher)
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int E, K, N, I;              // N output features, I inner features
    // FP8 form only
    const float *act_scale;      // row-major [cap, I/128], or [I/128][scale_ld] when scale_ld > 0
    const float *w_scale;        // [E, N/128, I/128]: one scale per 128 x 128 block of W_e
    int scale_ld;
};
struct GemmCombineArgs {
    GemmCombineParams p;
    const void *act;             // [cap, I] bf16 (or E4M3 codes when fp8), received-row layout
    const void *w;               // [E, N, I] bf16 (or E4M3 codes when fp8)
    void *out;                   // [T, N] bf16
    int64_t cap;
    int T;
    bool fp8;
};
// memset of the accumulator, the GEMM (one CTA per SM, num_sms CTAs) and the bf16 rounding
cudaError_t launch_gemm_combine(const GemmCombineArgs &g, int num_sms, cudaStream_t s);

// ---------------------------------------------------------------------------
// Layout fused with the dispatch (dispatch_lb.cu): a counts pre-pass over
// super-chunks, then a dispatch whose CTAs take token chunks by ticket, rank
// their pairs and find each chunk's place by decoupled look-back.
// ---------------------------------------------------------------------------
constexpr int kLbSuper = 16;          // token chunks per super-chunk (one pre-pass CTA each)
constexpr int kLbMaxPairs = 4096;     // (token, k) pairs per chunk at most
constexpr int kLbMaxTokens = 1 << 22; // tokens per call of the chunked kernel, below this

// Device-side control words of the fused path (in the handle's allocation,
// zeroed at creation; each kernel leaves them as it found them).
struct LbControl {
    unsigned int pre_arrivals;   // pre-pass CTAs that published their histogram (reset by the last)
    unsigned int ticket;         // next chunk to take (reset by the last dispatch CTA)
    unsigned int done;           // dispatch CTAs finished (reset by the last)
    unsigned int units;          // next batch of row parts to copy (dynamic copy; reset by the last)
    unsigned int pads;           // next expert whose padding rows to write (reset by the last)
    unsigned int epoch;          // tag of the last completed dispatch launch (look-back flags)
};

struct LbPlan {
    int nchunks;                 // token chunks
    int tpc;                     // tokens per chunk
    int nsuper;                  // super-chunks = pre-pass CTAs
};
LbPlan plan_lb(int T, int K, int num_sms);

struct LbParams {
    const int64_t *topk_idx;     // [T, K]
    const float *topk_weights;   // [T, K] or null
    const void *x;               // [T, H] bf16
    void *recv;                  // [cap, H] bf16 or e4m3
    float *recv_scale;           // FP8: row-major [cap, H/128] or column-major [H/128][scale_ld]
    int scale_ld;                // 0: row-major scales
    // routing (the handle's arrays)
    int32_t *pos, *row_src, *row_slot;
    float *row_weight;
    int32_t *cnt, *rank_tok, *eoff, *roff;
    // caller copies of the counts and offsets (may be null)
    int32_t *u_cnt, *u_rank_tok, *u_eoff, *u_roff;
    uint8_t *u_in_rank;
    // scratch
    int32_t *super_hist;         // [nsuper][E+R] pre-pass histograms
    int32_t *super_base;         // [nsuper][E] pairs of each expert in earlier super-chunks
    unsigned long long *flags;   // [nchunks][E] look-back words
    unsigned int *ready;         // [nchunks] launch tag once the chunk's routing is written
    LbControl *ctl;
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int stall_first_chunk;       // test hook: chunk 0 never publishes, so its successors' waits run out
    int T, K, E, R, L, A, H, id_bits;
    int nchunks, tpc, nsuper;
    int lb;                      // 1: the layout is computed in the kernel; 0: positions from pos
    int splits;                  // row parts per token (units per token)
    int chunk_bytes;             // bytes of x per unit
    int stages;                  // ring depth
    int prefetch_x;              // 1: the chunk's x rows are prefetched into L2 at its start
    int vec32;                   // FP8: 1 when recv is 32-byte aligned (32-byte code stores)
    int dyn;                     // 1: row parts are claimed in batches from ctl->units (K % 4 == 0)
    int dyn_batch;               // row parts per claim
};
cudaError_t launch_layout_counts(const LbParams &p, cudaStream_t s);
// The fused (lb = 1) or handle-driven (lb = 0) chunked dispatch, bf16 or FP8.
cudaError_t launch_dispatch_lb(const LbParams &p, bool fp8, int num_sms, cudaStream_t s);
cudaError_t dispatch_lb_prepare();

// Layout launch shape: the cluster kernel (G CTAs in one thread-block
// cluster, exchange through distributed shared memory) when a CTA can hold
// its share of the pairs, else the cooperative kernel (G CTAs, one grid-wide
// wait, chunk histograms in global scratch).
struct LayoutPlan {
    bool cluster;
    int G;
    int tokens_per_chunk;
    size_t smem;
};
constexpr int kClusterPairsTarget = 2048;   // target (token, k) pairs per cluster CTA
// Per device, before the first layout launch (kernel attributes, the
// largest co-schedulable cluster).
cudaError_t layout_prepare(int device);
LayoutPlan plan_layout(int device, int T, int E, int R, int K, int num_sms);

// launchers (return cudaError_t of the launch)
cudaError_t launch_layout(const LayoutParams &p, const LayoutPlan &plan, cudaStream_t s);
size_t layout_smem_bytes(int E, int R);
const void *layout_kernel_ptr();
// Launchers size their persistent grid from the occupancy of the kernel
// instance they pick: min(units, resident blocks per SM x num_sms).
cudaError_t launch_dispatch_bf16(const DispatchParams &p, int num_sms, cudaStream_t s);
cudaError_t launch_dispatch_fp8(const DispatchParams &p, int num_sms, cudaStream_t s);
// Layout and dispatch in one launch for batches of fewer than two tokens per
// SM: one CTA per token (at most num_sms), each counting all pairs itself
// (dispatch.cu); p.x == nullptr: the layout alone.
cudaError_t launch_layout_dispatch_small(const DispatchParams &p, const LayoutParams &lp, bool fp8, int num_sms,
                                         cudaStream_t s);
// Low-latency static layout + copy in one launch (p.ll_M > 0).
cudaError_t launch_ll_dispatch(const DispatchParams &p, bool fp8, int num_sms, cudaStream_t s);
cudaError_t launch_combine(const CombineParams &p, int num_sms, cudaStream_t s);

// Error text for ep_last_error and the library's launch counter (ep_api.cu).
void record_error(const char *msg);
int record_cuda_error(cudaError_t e, const char *what);   // returns EP_ERR_CUDA
void count_launch();

// Resident blocks per SM of one kernel instance, cached per device ordinal
// (0 = not yet known); launchers keep one as a function-local static.
constexpr int kMaxDevices = 64;
struct OccupancyCache {
    int per_device[kMaxDevices];
};

// Resident blocks per SM of `kernel` at `threads` threads and `smem` dynamic
// shared memory on the current device, through the cache.  Entries are read
// and written atomically, so host threads may launch concurrently; two that
// race both compute the same value.
inline int blocks_per_sm(const void *kernel, int threads, size_t smem, OccupancyCache *cache) {
    int dev = -1;
    int *slot = nullptr;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) slot = &cache->per_device[dev];
    int v = slot ? __atomic_load_n(slot, __ATOMIC_RELAXED) : 0;
    if (v > 0) return v;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, threads, smem) != cudaSuccess || v < 1) v = 1;
    if (slot) __atomic_store_n(slot, v, __ATOMIC_RELAXED);
    return v;
}
inline int persistent_grid(int units, int per_sm, int num_sms) {
    const int g = per_sm * num_sms;
    return units < g ? units : g;
}

// ---------------------------------------------------------------------------
// Device helpers (inline PTX for cache hints, ordering and the timer)
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// 16-byte read-only load that does not allocate in L1 (streamed data).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_v2(void *p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" : : "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ unsigned int lanemask_lt() {
    unsigned int m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 32-byte load / store (sm_100 256-bit vector access); address 32-byte aligned.
struct alignas(32) u32x8 {
    unsigned int v[8];
};

__device__ __forceinline__ u32x8 ld_stream_v8(const void *p) {
    u32x8 r;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r.v[0]), "=r"(r.v[1]), "=r"(r.v[2]), "=r"(r.v[3]), "=r"(r.v[4]), "=r"(r.v[5]),
                   "=r"(r.v[6]), "=r"(r.v[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v8(void *p, const u32x8 &r) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :
                 : "l"(p), "r"(r.v[0]), "r"(r.v[1]), "r"(r.v[2]), "r"(r.v[3]), "r"(r.v[4]), "r"(r.v[5]),
                   "r"(r.v[6]), "r"(r.v[7])
                 : "memory");
}

// ---- shared-memory barriers and bulk (non-tensor) async copies ------------
// Only CTA-local forms are used: no cluster multicast anywhere.
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" : : "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :
                 : "r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" : : "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete, at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

// global -> shared bulk copy completing on an mbarrier (16-byte aligned, size % 16 == 0)
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :
        : "r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// shared -> global bulk copy in the current bulk group
__device__ __forceinline__ void bulk_s2g(void *gdst, const void *smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :
                 : "l"(gdst), "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}

// L2 cache policies (fraction 1.0) for the .L2::cache_hint operand
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Bulk prefetch of global memory into L2 (16-byte aligned, size % 16 == 0)
// with an eviction-priority policy.
__device__ __forceinline__ void bulk_prefetch_l2(const void *gsrc, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;"
                 :
                 : "l"(gsrc), "r"(bytes), "l"(pol)
                 : "memory");
}

// 32-byte store with an L2 eviction-priority policy.
__device__ __forceinline__ void st_v8_policy(void *p, const u32x8 &r, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;"
                 :
                 : "l"(p), "r"(r.v[0]), "r"(r.v[1]), "r"(r.v[2]), "r"(r.v[3]), "r"(r.v[4]), "r"(r.v[5]),
                   "r"(r.v[6]), "r"(r.v[7]), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_v4_policy(void *p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;"
                 :
                 : "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" : : : "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" : : "n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" : : : "memory"); }

// Programmatic dependent launch.  A kernel launched with programmatic
// stream serialization may start while the kernel before it on the stream
// is still running; griddepcontrol.wait blocks the calling thread until that
// kernel has completed and its writes are visible, so every thread calls it
// before its first read of global memory.  launch_dependents lets such a
// dependent launch begin before this grid ends.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" : : : "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" : :); }

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (bulk copy) reads of them.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" : : : "memory");
}

// Exclusive scan of a[0..n) in shared memory, in place, by a CTA of
// kLayoutThreads threads; returns the total.  Caller must have synchronised
// after writing a[].
__device__ __forceinline__ int block_exclusive_scan(int32_t *a, int n, int32_t *s_tmp /*[kLayoutWarps+1]*/) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kLayoutThreads - 1) / kLayoutThreads;
    const int b = min(n, tid * per), e = min(n, b + per);
    int sum = 0;
    for (int i = b; i < e; ++i) sum += a[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kLayoutWarps ? s_tmp[lane] : 0;
        int iv = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, iv, o);
            if (lane >= o) iv += u;
        }
        if (lane < kLayoutWarps) s_tmp[lane] = iv - v;
        if (lane == 31) s_tmp[kLayoutWarps] = iv;
    }
    __syncthreads();
    int run = s_tmp[warp] + incl - sum;
    for (int i = b; i < e; ++i) {
        int v = a[i];
        a[i] = run;
        run += v;
    }
    const int total = s_tmp[kLayoutWarps];
    __syncthreads();
    return total;
}

// bf16 pair in a 32-bit word -> two floats (exact)
__device__ __forceinline__ float bf16_lo(unsigned int u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(unsigned int u) { return __uint_as_float(u & 0xffff0000u); }

}  // namespace ep

// The opaque handle.
struct ep_handle {
    ep_config cfg;
    int device;
    int num_sms;
    int l2_bytes;                   // the device's L2 size
    int64_t cap;
    // layout launch shape
    ep::LayoutPlan plan;
    int G;
    int tokens_per_chunk;
    // one device allocation, carved
    void *block;
    size_t block_bytes;
    int32_t *pos, *row_src, *row_slot;
    float *row_weight;
    int32_t *cnt, *rank_tok, *eoff, *roff;
    int32_t *chunk_counts;
    ep::GridBarrier *barrier;
    unsigned int *status;
    bool has_layout;
    int sm_limit;                   // SMs dispatch / combine may occupy (0: all)
    int scale_layout;               // EP_SCALES_*
    int ll_M;                       // > 0: low-latency handle with ll_M slots per expert
    unsigned long long wait_limit_ns;
    int barrier_extra;
    // fused layout + dispatch
    ep::LbPlan lb;
    ep::LbControl *lb_ctl;
    int32_t *lb_super_hist, *lb_super_base;
    unsigned long long *lb_flags;
    unsigned int *lb_ready;
};
