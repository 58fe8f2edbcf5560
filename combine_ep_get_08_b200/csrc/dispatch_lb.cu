// dispatch_lb.cu -- the layout fused with the dispatch (sm_100a).
//
// ep_layout_dispatch / ep_layout_dispatch_fp8 compute exactly what
// ep_get_layout followed by ep_dispatch / ep_dispatch_fp8 computes, in two
// launches that overlap:
//
//   layout_counts_kernel   one CTA per super-chunk of kLbSuper token chunks:
//     the expert and distinct-rank histograms of its tokens and their
//     is_token_in_rank rows.  The last CTA to arrive (an arrival counter,
//     nobody waits) adds the histograms up, forms the padded expert offsets
//     (expert_alignment, bowenzhou.top "deepep/01-overview" section 1.1) and,
//     for each super-chunk, how many pairs of each expert earlier
//     super-chunks hold.
//
//   dispatch_lb_kernel     one CTA per SM.  CTAs take token chunks in launch
//     order from an atomic ticket.  A chunk's pairs are ranked with warp
//     ballots, so that inside an expert the rows follow (token, k) order --
//     the order in which the moe_dispatch loop of the "lesson14_deepep"
//     practice task appends tokens to each expert's queue.  The chunk then
//     publishes its per-expert counts and finds how many pairs of each
//     expert the earlier chunks of its super-chunk hold by decoupled
//     look-back (the single-pass scan of Merrill and Garland, "Single-pass
//     Parallel Prefix Scan with Decoupled Look-back", 2016): each chunk
//     publishes first its own count (an aggregate) and, once known, its
//     running total (an inclusive prefix); a chunk reads its predecessors'
//     words back to the first running total.  Chunks are taken in launch
//     order and publish their aggregate before they wait, so every wait is
//     on a chunk whose CTA is running and will publish without waiting; every
//     wait is bounded by %globaltimer (EP_DEV_WAIT_TIMEOUT).  All of this
//     reads only topk_idx, so it runs before the dependency wait, beside the
//     pre-pass.  After it, a pair's row is the expert's offset + the pairs of
//     earlier super-chunks + the look-back prefix + its rank; the chunk's
//     routing is written and a per-chunk ready flag released.  Then the CTAs
//     copy: each claims row parts in small batches from an atomic counter (a
//     part waits, bounded, for the ready flag of its token's chunk), and the
//     x bytes and the token's destinations stream through a shared-memory
//     ring of bulk copies (TMA engine, no multicast) to the token's K rows, as
//     a plain copy (bf16) or with the fused 1x128-block FP8 E4M3 quantisation
//     of "m.nlpx.cn/news/135159" section 4.1.  No CTA copies before it has
//     finished every chunk it took, so a copy waits only on chunks that
//     running CTAs complete without waiting on copies.  One warp writes the
//     padding rows (zeros, and -1 routing) with bulk copies meanwhile.
//
// With lb = 0 the same kernel takes the positions from the handle (a layout
// computed earlier): it is the dispatch of ep_dispatch / ep_dispatch_fp8 for
// batches that fill the GPU.
#include "ep_internal.cuh"
#include "fp8_block.cuh"

#ifndef EP_LB_FP8_GROUPS
#define EP_LB_FP8_GROUPS 2          // FP8 consumer groups per CTA (quantisation needs more warps)
#endif
// Fused path, x into L2: 0 never, 1 after the dependency wait, 2 after this
// CTA's layout phase.  Layout then dispatch span (two runs each): dsv3 bf16
// 102.4 / 103.3 / 98.9 us for 0 / 1 / 2; skew FP8 90.7 / 93.7 / 95.8 us;
// large FP8 229.3 / 229.3 / 229.1 us.
#ifndef EP_LB_FUSED_PREFETCH_BF16
#define EP_LB_FUSED_PREFETCH_BF16 2
#endif
#ifndef EP_LB_FUSED_PREFETCH_FP8
#define EP_LB_FUSED_PREFETCH_FP8 0
#endif
// Positions from the handle (lb = 0), x into L2: 0 never, 1 before the
// dependency wait (overlapping the layout kernel), 2 after it (padding warp).
// Two runs each, layout-then-dispatch span / dispatch alone: dsv3 bf16
// 99.6 / 92.3 us (1), 102.3 / 91.5 (0), 101.3 / 90.1 (2); skew FP8 97.0 /
// 83.0 (1), 98.7 / 84.5 (0), 99.7 / 84.3 (2).  The span is what a step pays.
#ifndef EP_LB_NORMAL_PREFETCH_BF16
#define EP_LB_NORMAL_PREFETCH_BF16 1
#endif
#ifndef EP_LB_NORMAL_PREFETCH_FP8
#define EP_LB_NORMAL_PREFETCH_FP8 1
#endif
// lb = 0: claim the first row parts and load their x before the dependency
// wait.  Two runs each, dispatch alone / layout-then-dispatch span: skew FP8
// 81.0 / 95.9 us with, 82.8 / 97.7 us without; dsv3 bf16 96.7 / 100.6 us with,
// 93.0 / 98.9 us without.
#ifndef EP_LB_PREISSUE_BF16
#define EP_LB_PREISSUE_BF16 0
#endif
#ifndef EP_LB_PREISSUE_FP8
#define EP_LB_PREISSUE_FP8 1
#endif
#ifndef EP_LB_RING_BYTES
#define EP_LB_RING_BYTES (112 * 1024)
#endif

namespace ep {

namespace {

constexpr int kGroupWarps = 7;          // warps per consumer group
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kLayoutRankWarps = 8;     // warps that rank a chunk's pairs
constexpr int kMaxStages = 16;
constexpr int kZeroBytes = 8192;        // zeroed shared memory the padding warp copies from
constexpr int kFp8Ept = 32;             // FP8: bf16 elements per consumer thread
constexpr int kStageDst = kMaxTopk + 4;  // int32 per stage for a token's destinations (+ alignment lead)
#ifndef EP_LB_DYN_TOKENS_BF16
#define EP_LB_DYN_TOKENS_BF16 1     // tokens per claim of the dynamic copy, bf16 (dsv3: 1 -> 90.8 us,
#endif                              // 2 -> 92.4 us, 4 -> 94.7 us)
#ifndef EP_LB_DYN_TOKENS_FP8
#define EP_LB_DYN_TOKENS_FP8 1      // tokens per claim, FP8 (skew: 1 -> 84.9 us, 2 -> 86.0, 4 -> 87.2,
#endif                              // 8 -> 86.7; large: 212.0, 214.4, 217.5, 221.5)

template <int G>
struct Shape {
    static constexpr int kSetThreads = 32 + G * kGroupThreads;   // producer warp + consumer groups
    static constexpr int kThreads = kSetThreads + 32;            // + the padding warp
    static constexpr int kPadWarp = kThreads / 32 - 1;
};

__host__ __device__ __forceinline__ size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Dynamic shared memory carve-up (same on host and device).
struct Carve {
    size_t ring, bars, zeros, e16, rk16, cnt, base, agg, unit, stpos, total;
};
__host__ __device__ __forceinline__ Carve carve(int stages, int chunk_bytes, int E) {
    Carve c;
    size_t o = 0;
    c.ring = o;  o += up((size_t)stages * chunk_bytes, 128);
    c.bars = o;  o += 2 * kMaxStages * sizeof(uint64_t);
    c.zeros = o; o += kZeroBytes;
    c.e16 = o;   o += (size_t)kLbMaxPairs * sizeof(int16_t);
    c.rk16 = o;  o += (size_t)kLbMaxPairs * sizeof(int16_t);
    c.cnt = o;   o += (size_t)kLayoutRankWarps * (E + 1) * sizeof(int32_t);
    c.base = o;  o += (size_t)E * sizeof(int32_t);
    c.agg = o;   o += (size_t)E * sizeof(int32_t);
    o = up(o, 128);
    c.unit = o;  o += (size_t)kMaxStages * sizeof(int32_t);
    o = up(o, 128);                      // bulk-copy destinations: 16-byte aligned
    c.stpos = o; o += (size_t)kMaxStages * kStageDst * sizeof(int32_t);
    c.total = up(o, 128);
    return c;
}

// named barrier 1: the producer warp and the consumer groups (the padding
// warp runs on its own and never takes part)
__device__ __forceinline__ void set_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" : : "r"(nthreads) : "memory");
}

// Look-back word of (chunk, expert): the count in the low 32 bits; the high
// 32 bits are tag << 1 | inclusive, tag = the launch's epoch tag (1 ..
// 2^31 - 1), so zeroed words and words of earlier launches read as "not
// published yet".
__device__ __forceinline__ unsigned long long lb_word(unsigned int tag, bool inclusive, int v) {
    return ((unsigned long long)((tag << 1) | (inclusive ? 1u : 0u)) << 32) | (unsigned int)v;
}
__device__ __forceinline__ unsigned int lb_tag(unsigned long long w) { return (unsigned int)(w >> 33); }
__device__ __forceinline__ bool lb_inclusive(unsigned long long w) { return (w >> 32) & 1ull; }

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" : : "l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Orders generic-proxy global memory accesses this thread has observed
// before its later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" : : : "memory");
}

__device__ __forceinline__ void st_release_u32(unsigned int *p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" : : "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ bool valid_id(int64_t e, int E) { return e >= 0 && e < E; }

__device__ __forceinline__ int64_t scale_at(const LbParams &p, int row, int b, int NB) {
    return p.scale_ld == 0 ? (int64_t)row * NB + b : (int64_t)b * p.scale_ld + row;
}

// ---------------------------------------------------------------------------
// Counts pre-pass
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads, 1) layout_counts_kernel(LbParams p) {
    extern __shared__ int32_t smem_c[];
    const int E = p.E, R = p.R, K = p.K, L = p.L, ncols = E + R;
    int32_t *s_hist = smem_c;            // [E+R] this super-chunk's counts, later the totals
    int32_t *s_eoff = s_hist + ncols;    // [E+1] padded expert offsets
    __shared__ int32_t s_tmp[kLayoutWarps + 1];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    pdl_launch_dependents();             // the dispatch may start its own layout work now

    const int tps = p.tpc * kLbSuper;
    const int t0 = min(p.T, (int)blockIdx.x * tps), t1 = min(p.T, t0 + tps);
    for (int j = tid; j < ncols; j += kLayoutThreads) s_hist[j] = 0;
    __syncthreads();
    for (int64_t q = (int64_t)t0 * K + tid; q < (int64_t)t1 * K; q += kLayoutThreads) {
        const int64_t e = __ldg(p.topk_idx + q);
        if (valid_id(e, E))
            atomicAdd(&s_hist[e], 1);
        else if (e != -1)
            atomicOr(p.status, EP_DEV_BAD_EXPERT);   // -1: a masked top-k slot
    }
    // distinct ranks of each token, and its is_token_in_rank row
    for (int t = t0 + tid; t < t1; t += kLayoutThreads) {
        const int64_t *row = p.topk_idx + (int64_t)t * K;
        uint8_t *dst = p.u_in_rank ? p.u_in_rank + (int64_t)t * R : nullptr;
        if (R <= 64) {
            unsigned long long mask = 0;
            for (int k = 0; k < K; ++k) {
                const int64_t e = __ldg(row + k);
                if (valid_id(e, E)) mask |= 1ull << (int)(e / L);
            }
            for (unsigned long long m = mask; m; m &= m - 1) atomicAdd(&s_hist[E + __ffsll((long long)m) - 1], 1);
            if (dst)
                for (int r = 0; r < R; ++r) dst[r] = (uint8_t)((mask >> r) & 1ull);
        } else {
            if (dst)
                for (int r = 0; r < R; ++r) dst[r] = 0;
            for (int k = 0; k < K; ++k) {
                const int64_t e = __ldg(row + k);
                if (!valid_id(e, E)) continue;
                const int r = (int)(e / L);
                bool dup = false;
                for (int k2 = 0; k2 < k; ++k2) {
                    const int64_t e2 = __ldg(row + k2);
                    if (valid_id(e2, E) && (int)(e2 / L) == r) dup = true;
                }
                if (!dup) atomicAdd(&s_hist[E + r], 1);
                if (dst) dst[r] = 1;
            }
        }
    }
    __syncthreads();
    int32_t *mine = p.super_hist + (size_t)blockIdx.x * ncols;
    for (int j = tid; j < ncols; j += kLayoutThreads) mine[j] = s_hist[j];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.ctl->pre_arrivals, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;

    // the last CTA: every histogram is published.  Per column, the totals and
    // (experts) the pairs in earlier super-chunks, eight loads in flight
    __threadfence();
    const int ns = gridDim.x;
    for (int j = tid; j < ncols; j += kLayoutThreads) {
        int tot = 0;
        for (int s0 = 0; s0 < ns; s0 += 8) {
            int v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = s0 + k < ns ? __ldcg(p.super_hist + (size_t)(s0 + k) * ncols + j) : 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (j < E && s0 + k < ns) p.super_base[(size_t)(s0 + k) * E + j] = tot;
                tot += v[k];
            }
        }
        s_hist[j] = tot;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kLayoutThreads) s_eoff[e] = (s_hist[e] + p.A - 1) / p.A * p.A;
    __syncthreads();
    const int rows = block_exclusive_scan(s_eoff, E, s_tmp);
    if (tid == 0) s_eoff[E] = rows;
    __syncthreads();
    for (int e = tid; e < E; e += kLayoutThreads) {
        p.cnt[e] = s_hist[e];
        if (p.u_cnt) p.u_cnt[e] = s_hist[e];
    }
    for (int e = tid; e <= E; e += kLayoutThreads) {
        p.eoff[e] = s_eoff[e];
        if (p.u_eoff) p.u_eoff[e] = s_eoff[e];
    }
    for (int r = tid; r < R; r += kLayoutThreads) {
        p.rank_tok[r] = s_hist[E + r];
        if (p.u_rank_tok) p.u_rank_tok[r] = s_hist[E + r];
    }
    for (int r = tid; r <= R; r += kLayoutThreads) {
        p.roff[r] = s_eoff[r * L];
        if (p.u_roff) p.u_roff[r] = s_eoff[r * L];
    }
    if (tid == 0) atomicExch(&p.ctl->pre_arrivals, 0u);   // every CTA has arrived: ready for the next launch
}

// ---------------------------------------------------------------------------
// Padding rows: the padding warps claim experts from a counter and their 32
// lanes share each expert's padding rows (rows eoff[e] + cnt[e] ..
// eoff[e+1]); every row is written with bulk
// shared->global copies of a zeroed block: a zero bf16 row, or zero codes and
// (row-major, when 16-byte sized) zero scales; with lb = 1 also its routing
// (row_src = row_slot = -1, row_weight = 0).  Before that, in the fused path
// (lb = 1) with prefetch_x, lane 0 may pull this CTA's share of x into L2,
// issued late enough not to delay the latency-bound layout work (bf16: once
// this CTA's layout phase is over; FP8: not at all, which measured faster).
// ---------------------------------------------------------------------------
template <bool FP8>
__device__ __forceinline__ void pad_rows(const LbParams &p, const uint8_t *zeros, int lane, int n_cta, int chunk,
                                         volatile int *rows_done) {
    pdl_wait();   // offsets and counts come from the kernel before
    constexpr int kPrefetch = FP8 ? EP_LB_FUSED_PREFETCH_FP8 : EP_LB_FUSED_PREFETCH_BF16;
    constexpr int kPrefetchNormal = FP8 ? EP_LB_NORMAL_PREFETCH_FP8 : EP_LB_NORMAL_PREFETCH_BF16;
    if (kPrefetchNormal == 2 && !p.lb && p.prefetch_x && lane == 0) {
        const uint64_t pol_x = policy_evict_last();
        const uint8_t *x = static_cast<const uint8_t *>(p.x);
        for (int i = 0; i < n_cta; ++i) {
            const int u = (int)blockIdx.x + i * (int)gridDim.x, t = u / p.splits, part = u - t * p.splits;
            bulk_prefetch_l2(x + (int64_t)t * 2 * p.H + (int64_t)part * chunk, (uint32_t)chunk, pol_x);
        }
    }
    if (kPrefetch == 2 && p.lb && p.prefetch_x && lane == 0) {
        // after this CTA's layout phase has published its rows (the flag is set
        // on an abort too; bounded all the same)
        const unsigned long long t0 = globaltimer_ns();
        while (!*rows_done && globaltimer_ns() - t0 < p.wait_limit_ns) {
        }
    }
    if (kPrefetch && p.lb && p.prefetch_x && lane == 0) {
        const uint64_t pol_x = policy_evict_last();
        const uint8_t *x = static_cast<const uint8_t *>(p.x);
        for (int i = 0; i < n_cta; ++i) {
            const int u = (int)blockIdx.x + i * (int)gridDim.x, t = u / p.splits, part = u - t * p.splits;
            bulk_prefetch_l2(x + (int64_t)t * 2 * p.H + (int64_t)part * chunk, (uint32_t)chunk, pol_x);
        }
    }
    if (p.A <= 1) return;
    const int row_bytes = FP8 ? p.H : 2 * p.H;
    const int NB = p.H / 128;
    const bool bulk_scales = FP8 && p.scale_ld == 0 && (NB * 4) % 16 == 0 &&
                             (reinterpret_cast<uintptr_t>(p.recv_scale) & 15) == 0;
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    // experts are claimed one at a time from a counter: padding per expert is
    // 0 .. A-1 rows, and a fixed assignment (experts b, b + G, ...) measured
    // skew FP8 85.4 -> 83.3 us against this
    for (;;) {
        int e = 0;
        if (lane == 0) e = (int)atomicAdd(&p.ctl->pads, 1u);
        e = __shfl_sync(0xffffffffu, e, 0);
        if (e >= p.E) break;
        const int r0 = __ldcg(p.eoff + e) + __ldcg(p.cnt + e), r1 = __ldcg(p.eoff + e + 1);
        for (int r = r0 + lane; r < r1; r += 32) {
            if (p.lb) {
                p.row_src[r] = -1;
                p.row_slot[r] = -1;
                if (p.topk_weights) p.row_weight[r] = 0.0f;
            }
            uint8_t *o = recv + (int64_t)r * row_bytes;
            for (int off = 0; off < row_bytes; off += kZeroBytes)
                bulk_s2g(o + off, zeros, (uint32_t)min(kZeroBytes, row_bytes - off));
            if (FP8) {
                if (bulk_scales)
                    bulk_s2g(p.recv_scale + (int64_t)r * NB, zeros, (uint32_t)(NB * 4));
                else
                    for (int b = 0; b < NB; ++b) p.recv_scale[scale_at(p, r, b, NB)] = 0.0f;
            }
        }
        bulk_commit();
    }
    bulk_wait_all();
}

// bf16 unit: copy the staged part of a token row to its K rows.
template <int VB>
__device__ __forceinline__ void copy_unit(const LbParams &p, const uint8_t *src, const int32_t *dsts, int part,
                                          int gtid, uint64_t pol) {
    const int row_bytes = 2 * p.H, chunk = p.chunk_bytes, nv = chunk / VB;
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    for (int v = gtid; v < nv; v += kGroupThreads) {
        if constexpr (VB == 32) {
            const uint4 a = *reinterpret_cast<const uint4 *>(src + v * 32);
            const uint4 b = *reinterpret_cast<const uint4 *>(src + v * 32 + 16);
            u32x8 val;
            val.v[0] = a.x; val.v[1] = a.y; val.v[2] = a.z; val.v[3] = a.w;
            val.v[4] = b.x; val.v[5] = b.y; val.v[6] = b.z; val.v[7] = b.w;
            for (int k = 0; k < p.K; ++k) {
                const int dst = dsts[k];
                if (dst >= 0) st_v8_policy(recv + (int64_t)dst * row_bytes + (int64_t)part * chunk + v * 32, val, pol);
            }
        } else {
            const uint4 val = *reinterpret_cast<const uint4 *>(src + v * 16);
            for (int k = 0; k < p.K; ++k) {
                const int dst = dsts[k];
                if (dst >= 0) st_v4_policy(recv + (int64_t)dst * row_bytes + (int64_t)part * chunk + v * 16, val, pol);
            }
        }
    }
}

// FP8 unit: thread gtid quantises elements [gtid*32, gtid*32+32) of the
// staged part (4 consecutive lanes per 1x128 block) and stores the 32 code
// bytes to each of the K rows; the block's first lane stores its scale.
__device__ __forceinline__ void quantise_unit(const LbParams &p, const uint8_t *src, const int32_t *dsts, int part,
                                              int gtid, uint64_t pol) {
    constexpr int TPB = 128 / kFp8Ept, NW = kFp8Ept / 2;
    const int U = p.chunk_bytes / 2;           // elements per unit (a multiple of 128)
    const bool act = gtid * kFp8Ept < U;       // whole blocks of 4 lanes are active or idle
    unsigned int w[NW];
    if (act) {
#pragma unroll
        for (int i = 0; i < NW / 4; ++i) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + gtid * 2 * kFp8Ept + 16 * i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) w[i] = 0;
    }
    unsigned int q[8];
    const float scale = quantize_block<TPB, NW>(w, q);   // every lane of the warp takes part
    if (!act) return;
    const int col = part * U + gtid * kFp8Ept;
    const int NB = p.H / 128, b = col / 128;
    const bool lead = (gtid % TPB) == 0;
    u32x8 v;
#pragma unroll
    for (int i = 0; i < 8; ++i) v.v[i] = q[i];
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    for (int k = 0; k < p.K; ++k) {
        const int dst = dsts[k];
        if (dst < 0) continue;
        uint8_t *o = recv + (int64_t)dst * p.H + col;
        if (p.vec32) {
            st_v8_policy(o, v, pol);
        } else {   // a 16-byte aligned buffer
            st_v4_policy(o, make_uint4(q[0], q[1], q[2], q[3]), pol);
            st_v4_policy(o + 16, make_uint4(q[4], q[5], q[6], q[7]), pol);
        }
        if (lead) p.recv_scale[scale_at(p, dst, b, NB)] = scale;
    }
}

template <int VB, bool FP8, int G>
__global__ void __launch_bounds__(Shape<G>::kThreads, 1) dispatch_lb_kernel(LbParams p) {
    using S = Shape<G>;
    constexpr int NSET = S::kSetThreads;
    extern __shared__ __align__(128) uint8_t smem[];
    const Carve cv = carve(p.stages, p.chunk_bytes, p.E);
    uint8_t *ring = smem + cv.ring;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + cv.bars);
    uint64_t *empty = full + kMaxStages;
    uint8_t *zeros = smem + cv.zeros;
    int16_t *s_e = reinterpret_cast<int16_t *>(smem + cv.e16);
    int16_t *s_rk = reinterpret_cast<int16_t *>(smem + cv.rk16);
    int32_t *s_cnt = reinterpret_cast<int32_t *>(smem + cv.cnt);
    int32_t *s_base = reinterpret_cast<int32_t *>(smem + cv.base);
    int32_t *s_agg = reinterpret_cast<int32_t *>(smem + cv.agg);
    int32_t *s_unit = reinterpret_cast<int32_t *>(smem + cv.unit);     // [stages] row part | lead << 28 (-1: end)
    int32_t *s_stpos = reinterpret_cast<int32_t *>(smem + cv.stpos);   // [stages][kStageDst] its destinations
    __shared__ int s_ticket;
    __shared__ int s_abort;
    __shared__ int s_rows_done;   // this CTA's layout phase is over (its rows published, or aborted)
    __shared__ unsigned int s_tag;
    volatile int *abort_flag = &s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.E, K = p.K, ES = E + 1, NS = p.stages, chunk = p.chunk_bytes;
    const int row_bytes = 2 * p.H;   // bytes of an x row
    const bool padding = p.A > 1;
    const uint8_t *x = static_cast<const uint8_t *>(p.x);

    if (padding) {
        for (int i = tid; i < kZeroBytes / 16; i += S::kThreads) reinterpret_cast<uint4 *>(zeros)[i] = make_uint4(0, 0, 0, 0);
        fence_async_smem();
    }
    // this CTA's share of the row parts for the L2 prefetch of x: b, b + G, ...
    const int GC = gridDim.x;
    const int total_units = p.T * p.splits;
    const int n_cta = total_units > (int)blockIdx.x ? (total_units - (int)blockIdx.x + GC - 1) / GC : 0;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGroupWarps);
        }
        fence_async_smem();
        s_abort = 0;
        s_rows_done = 0;
        // the previous launch's tag is stable: it changes only after every CTA
        // of that launch finished, and that launch completed before this one
        s_tag = (__ldcg(&p.ctl->epoch) % 0x7fffffffu) + 1u;
    }
    __syncthreads();

    if (warp == S::kPadWarp) {
        pad_rows<FP8>(p, zeros, lane, n_cta, chunk, &s_rows_done);
    } else {
        const uint64_t pol_out = policy_evict_first();
        const unsigned int tag = s_tag;
        int issued = 0;   // producer (thread 0): row parts whose load was issued
        // the first chunk's ticket is requested before anything else
        if (p.lb && tid == 0) s_ticket = (int)atomicAdd(&p.ctl->ticket, 1u);
        // x is an input: with lb = 0 a share of it (row parts b, b + G, ... --
        // together all of x) goes into L2 now, overlapping the kernel before;
        // with lb = 1 the padding warp does that after the dependency wait,
        // where it cannot delay the latency-bound layout phases
        if (tid == 0 && p.prefetch_x && !p.lb && (FP8 ? EP_LB_NORMAL_PREFETCH_FP8 : EP_LB_NORMAL_PREFETCH_BF16) == 1) {
            const uint64_t pol_x = policy_evict_last();
            for (int i = 0; i < n_cta; ++i) {
                const int u = (int)blockIdx.x + i * GC, t = u / p.splits, part = u - t * p.splits;
                bulk_prefetch_l2(x + (int64_t)t * row_bytes + (int64_t)part * chunk, (uint32_t)chunk, pol_x);
            }
        }
        __syncwarp();

        // ---- phase 1: the layout of every chunk this CTA takes ----
        for (bool first = true; p.lb; first = false) {
            set_sync(NSET);
            if (tid == 0 && !first) s_ticket = (int)atomicAdd(&p.ctl->ticket, 1u);
            set_sync(NSET);
            const int c = s_ticket;
            if (c >= p.nchunks || *abort_flag) break;
            const int t0 = c * p.tpc, t1 = min(p.T, t0 + p.tpc);
            const int nt = t1 - t0, n = nt * K;
            const int64_t q0 = (int64_t)t0 * K;
            const int ppw = (n + kLayoutRankWarps * 32 - 1) / (kLayoutRankWarps * 32) * 32;   // pairs per ranking warp
            // ranks: warp w walks pairs [w*ppw, (w+1)*ppw) 32 at a time; a lane's
            // rank is its warp's running count of its expert plus the lanes below
            // it with the same expert (ballots over the id bits)
            if (warp < kLayoutRankWarps) {
                int32_t *wrow = s_cnt + warp * ES;
                for (int e = lane; e < ES; e += 32) wrow[e] = 0;
                __syncwarp();
                const int lo = warp * ppw, hi = min(n, lo + ppw);
                for (int j0 = lo; j0 < hi; j0 += 32 * 8) {
                    int64_t v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int i = j0 + u * 32 + lane;
                        v[u] = i < hi ? __ldg(p.topk_idx + q0 + i) : (int64_t)-1;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (j0 + u * 32 >= hi) break;   // warp-uniform
                        const int i = j0 + u * 32 + lane;
                        const int e = valid_id(v[u], E) ? (int)v[u] : -1;
                        if (i < hi && e < 0 && v[u] != -1) atomicOr(p.status, EP_DEV_BAD_EXPERT);
                        unsigned int peers = __ballot_sync(0xffffffffu, e >= 0);
                        if (e < 0) peers = ~peers;
                        for (int bit = 0; bit < p.id_bits; ++bit) {
                            const int bv = (e >> bit) & 1;
                            const unsigned int bal = __ballot_sync(0xffffffffu, bv);
                            peers &= bv ? bal : ~bal;
                        }
                        const int lrank = __popc(peers & lanemask_lt());
                        const int base = e >= 0 ? wrow[e] : 0;
                        __syncwarp();
                        if (e >= 0 && lrank == 0) wrow[e] = base + __popc(peers);
                        __syncwarp();
                        if (i < hi) {
                            s_e[i] = (int16_t)e;
                            s_rk[i] = (int16_t)(base + lrank);
                        }
                    }
                }
            }
            set_sync(NSET);
            // each expert's counts become exclusive prefixes over the ranking
            // warps; their total is the chunk's aggregate
            for (int e = tid; e < E; e += NSET) {
                int run = 0;
#pragma unroll
                for (int w = 0; w < kLayoutRankWarps; ++w) {
                    const int vv = s_cnt[w * ES + e];
                    s_cnt[w * ES + e] = run;
                    run += vv;
                }
                s_agg[e] = run;
            }
            set_sync(NSET);
            // publish, then look back over the earlier chunks of the super-chunk
            const int c0 = c / kLbSuper * kLbSuper;
            unsigned long long *fl = p.flags;
            if (!(p.stall_first_chunk && c == 0))
                for (int e = tid; e < E; e += NSET)
                    st_relaxed_u64(fl + (size_t)c * E + e, lb_word(tag, c == c0, s_agg[e]));
            if (c > c0) {
                const int np = c - c0;   // predecessors, at most kLbSuper - 1
                for (int e = tid; e < E; e += NSET) {
                    unsigned long long v[kLbSuper - 1];
#pragma unroll
                    for (int k = 0; k < kLbSuper - 1; ++k)
                        v[k] = k < np ? ld_relaxed_u64(fl + (size_t)(c - 1 - k) * E + e) : 0ull;
                    int sum = 0;
                    bool ok = true;
#pragma unroll
                    for (int k = 0; k < kLbSuper - 1; ++k) {
                        if (k >= np) break;
                        unsigned long long wv = v[k];
                        if (lb_tag(wv) != tag) {   // not published yet: wait for it, bounded
                            const unsigned long long tw0 = globaltimer_ns();
                            for (;;) {
                                wv = ld_relaxed_u64(fl + (size_t)(c - 1 - k) * E + e);
                                if (lb_tag(wv) == tag) break;
                                if (globaltimer_ns() - tw0 > p.wait_limit_ns) {
                                    ok = false;
                                    break;
                                }
                            }
                            if (!ok) break;
                        }
                        sum += (int)(unsigned int)wv;
                        if (lb_inclusive(wv)) break;
                    }
                    if (!ok) {
                        atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *abort_flag = 1;
                    } else {
                        st_relaxed_u64(fl + (size_t)c * E + e, lb_word(tag, true, sum + s_agg[e]));
                    }
                    s_base[e] = sum;
                }
            } else {
                for (int e = tid; e < E; e += NSET) s_base[e] = 0;
            }
            set_sync(NSET);
            if (*abort_flag) break;
            if (first) pdl_wait();   // the pre-pass is complete and visible
            // rows: expert offset + this super-chunk's earlier pairs + the look-back
            // prefix + the rank inside the chunk
            const int sb = c / kLbSuper;
            for (int e = tid; e < E; e += NSET)
                s_base[e] += __ldcg(p.eoff + e) + __ldcg(p.super_base + (size_t)sb * E + e);
            set_sync(NSET);
            for (int i = tid; i < n; i += NSET) {
                const int e = s_e[i];
                int dst = -1;
                if (e >= 0) {
                    dst = s_base[e] + s_cnt[(i / ppw) * ES + e] + s_rk[i];
                    const int tl = i / K;
                    p.row_src[dst] = t0 + tl;
                    p.row_slot[dst] = i - tl * K;
                    if (p.topk_weights) p.row_weight[dst] = __ldg(p.topk_weights + q0 + i);
                }
                p.pos[q0 + i] = dst;
            }
            __threadfence();   // this thread's rows before the chunk's ready flag
            set_sync(NSET);
            if (tid == 0) st_release_u32(p.ready + c, tag);
        }
        // The producer's row parts: claimed in batches of dyn_batch from
        // ctl->units, one claim ahead (next_part() returns -1 when none is left).
        unsigned int claim_cur = 0, claim_next = 0;
        int part_u = 0, part_end = 0;
        auto next_part = [&]() -> int {
            for (;;) {
                if (part_u < part_end) return part_u++;
                if ((int64_t)claim_cur * p.dyn_batch >= total_units) return -1;
                claim_cur = claim_next;
                claim_next = atomicAdd(&p.ctl->units, 1u);
                part_u = (int)claim_cur * p.dyn_batch;
                part_end = min(total_units, part_u + p.dyn_batch);
                if (part_u >= total_units) return -1;
            }
        };
        // the destinations of part u: the 16-byte aligned span of pos that
        // holds its token's K entries (pos is followed by other arrays of the
        // handle's allocation, so the span never leaves it); the consumers skip
        // `lead` entries
        auto dst_span = [&](int u, int64_t *a0, int *lead, uint32_t *span) {
            const int64_t b0 = (int64_t)(u / p.splits) * K * 4;
            *a0 = b0 & ~(int64_t)15;
            *lead = (int)(b0 - *a0) / 4;
            *span = (uint32_t)((b0 + K * 4 - *a0 + 15) & ~(int64_t)15);
        };
        // x is an input and the claim counter belongs to the dispatch: with
        // positions from the handle (lb = 0) the producer claims its first
        // parts and fills the ring with their x bytes before the dependency
        // wait, overlapping the layout kernel; their destinations follow after it
        int pre = 0;
        if (tid == 0) {
            claim_cur = atomicAdd(&p.ctl->units, 1u);
            claim_next = atomicAdd(&p.ctl->units, 1u);
            part_u = (int)claim_cur * p.dyn_batch;
            part_end = min(total_units, part_u + p.dyn_batch);
            if (!p.lb && (FP8 ? EP_LB_PREISSUE_FP8 : EP_LB_PREISSUE_BF16)) {
                for (; pre < NS; ++pre) {
                    const int u = next_part();
                    if (u < 0) break;
                    int64_t a0;
                    int lead;
                    uint32_t span;
                    dst_span(u, &a0, &lead, &span);
                    const int t = u / p.splits, part = u - t * p.splits;
                    s_unit[pre] = u | (lead << 28);
                    mbar_arrive_expect_tx(&full[pre], (uint32_t)chunk + span);
                    bulk_g2s(ring + (size_t)pre * chunk, x + (int64_t)t * row_bytes + (int64_t)part * chunk, chunk,
                             &full[pre]);
                    ++issued;
                }
            }
        }
        __syncwarp();
        pdl_wait();            // (a no-op after the first wait) the layout before is complete and visible
        if (tid == 0) *static_cast<volatile int *>(&s_rows_done) = 1;

        // ---- phase 2: the copy; row parts claimed in batches of dyn_batch ----
        // The producer claims a batch from ctl->units (the next claim is
        // requested before the current batch is issued), and per row part puts
        // its x bytes and its token's K destinations (a second bulk copy) into
        // one stage, completing on the stage's barrier.  Consumer group grp takes
        // the stages g = grp, grp + G, ...; a part of -1 ends the group's loop.
        // CTAs on SMs that move bytes faster take more parts: against a fixed
        // interleaved order (CTA b taking parts b, b + G, ...) this measured
        // dsv3 bf16 96.1 -> 90.8 us and large FP8 (fused) 277.2 -> 237.1 us.
        {
            if (warp == 0) {
                if (lane == 0) {
                    // the destinations of the parts issued before the wait
                    for (int g = 0; g < pre; ++g) {
                        const int u = s_unit[g] & 0x0fffffff;
                        int64_t a0;
                        int lead;
                        uint32_t span;
                        dst_span(u, &a0, &lead, &span);
                        bulk_g2s(s_stpos + g * kStageDst, reinterpret_cast<const uint8_t *>(p.pos) + a0, span, &full[g]);
                    }
                    int g = pre;
                    for (;; ++g) {
                        if (*abort_flag) break;
                        const int u = next_part();
                        if (u < 0) break;
                        const int s = g % NS;
                        bool ok = g < NS || mbar_wait_bounded(&empty[s], ((g / NS) - 1) & 1, p.wait_limit_ns);
                        const int t = u / p.splits, part = u - t * p.splits;
                        if (ok && p.lb) {   // the chunk's rows are written (released by its CTA)
                            const unsigned int *rf = p.ready + t / p.tpc;
                            if (ld_acquire_u32(rf) != tag) {
                                const unsigned long long tw0 = globaltimer_ns();
                                while (ok && ld_acquire_u32(rf) != tag) ok = globaltimer_ns() - tw0 <= p.wait_limit_ns;
                            }
                            fence_proxy_async_global();   // those generic writes, before the bulk read below
                        }
                        if (!ok) {
                            atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                            *abort_flag = 1;
                            break;
                        }
                        int64_t a0;
                        int lead;
                        uint32_t span;
                        dst_span(u, &a0, &lead, &span);
                        s_unit[s] = u | (lead << 28);
                        mbar_arrive_expect_tx(&full[s], (uint32_t)chunk + span);
                        bulk_g2s(ring + (size_t)s * chunk, x + (int64_t)t * row_bytes + (int64_t)part * chunk, chunk,
                                 &full[s]);
                        bulk_g2s(s_stpos + s * kStageDst, reinterpret_cast<const uint8_t *>(p.pos) + a0, span, &full[s]);
                        ++issued;
                    }
                    // one end marker per consumer group
                    for (int k = 0; k < G && !*abort_flag; ++k, ++g) {
                        const int s = g % NS;
                        if (g >= NS && !mbar_wait_bounded(&empty[s], ((g / NS) - 1) & 1, p.wait_limit_ns)) {
                            atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                            *abort_flag = 1;
                            break;
                        }
                        s_unit[s] = -1;
                        mbar_arrive(&full[s]);
                    }
                }
                __syncwarp();
            } else {
                const int grp = (tid - 32) / kGroupThreads, gtid = (tid - 32) - grp * kGroupThreads;
                for (int g = grp;; g += G) {
                    const int s = g % NS;
                    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (g / NS) & 1, p.wait_limit_ns))) {
                        if (lane == 0) atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    const int su = s_unit[s];
                    if (su < 0) break;
                    const int u = su & 0x0fffffff, lead = su >> 28;
                    const int part = u % p.splits;
                    const int32_t *dsts = s_stpos + s * kStageDst + lead;
                    if constexpr (FP8)
                        quantise_unit(p, ring + (size_t)s * chunk, dsts, part, gtid, pol_out);
                    else
                        copy_unit<VB>(p, ring + (size_t)s * chunk, dsts, part, gtid, pol_out);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                }
            }
        }

        if (*abort_flag && tid == 0) {
            // let every issued load land before the CTA's shared memory goes away
            for (int j = max(0, issued - NS); j < issued; ++j)
                mbar_wait_bounded(&full[j % NS], (j / NS) & 1, p.wait_limit_ns);
        }
    }
    __syncthreads();
    if (tid == 0) {
        // the last CTA to finish leaves the control words ready for the next
        // launch: every CTA took its last ticket before it got here
        __threadfence();
        if (atomicAdd(&p.ctl->done, 1u) == gridDim.x - 1) {
            __threadfence();
            atomicExch(&p.ctl->ticket, 0u);
            atomicExch(&p.ctl->units, 0u);
            atomicExch(&p.ctl->pads, 0u);
            atomicExch(&p.ctl->done, 0u);
            atomicExch(&p.ctl->epoch, s_tag);
        }
    }
}

// Units per token and bytes per unit: bf16 rows split into the fewest
// power-of-two parts of at most 8 KB; FP8 rows into the fewest parts of at
// most 224 x 32 elements that hold whole 1x128 blocks.
bool lb_unit_shape(int H, bool fp8, int VB, int *splits, int *chunk_bytes) {
    if (fp8) {
        for (int sp = 1; sp <= H / 128; ++sp) {
            if (H % sp || (H / sp) % 128 || H / sp > kGroupThreads * kFp8Ept) continue;
            *splits = sp;
            *chunk_bytes = 2 * (H / sp);
            return true;
        }
        return false;
    }
    const int row_bytes = 2 * H;
    for (int sp = 1; sp <= 64; sp *= 2) {
        if (row_bytes % (sp * VB) || row_bytes / sp > 8192) continue;
        *splits = sp;
        *chunk_bytes = row_bytes / sp;
        return true;
    }
    return false;
}

template <typename Kern>
cudaError_t launch_pdl_lb(Kern kernel, int grid, int block, size_t smem, cudaStream_t s, const LbParams &p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

constexpr int kFp8Groups = EP_LB_FP8_GROUPS;

// Dynamic shared memory the chunked kernels may use on each device: the
// opt-in limit per block less their static shared memory (0: not set up).
int g_smem_limit[kMaxDevices];

size_t smem_limit() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    return (size_t)__atomic_load_n(&g_smem_limit[dev], __ATOMIC_ACQUIRE);
}

}  // namespace

LbPlan plan_lb(int T, int K, int num_sms) {
    LbPlan pl{};
    if (T <= 0) {
        pl.nchunks = 0;
        pl.tpc = 1;
        pl.nsuper = 1;
        return pl;
    }
    // about one chunk per SM, at most kLbMaxPairs pairs each
    const int64_t pairs = (int64_t)T * K;
    int64_t n = (pairs + kLbMaxPairs - 1) / kLbMaxPairs;
    if (n < num_sms) n = num_sms < T ? num_sms : T;
    int tpc = (int)((T + n - 1) / n);
    while ((int64_t)tpc * K > kLbMaxPairs && tpc > 1) --tpc;
    pl.tpc = tpc;
    pl.nchunks = (T + tpc - 1) / tpc;
    pl.nsuper = (pl.nchunks + kLbSuper - 1) / kLbSuper;
    return pl;
}

cudaError_t dispatch_lb_prepare() {
    int dev = -1, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (__atomic_load_n(&g_smem_limit[dev], __ATOMIC_ACQUIRE) > 0) return cudaSuccess;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    const void *kernels[] = {reinterpret_cast<const void *>(&dispatch_lb_kernel<32, false, 1>),
                             reinterpret_cast<const void *>(&dispatch_lb_kernel<16, false, 1>),
                             reinterpret_cast<const void *>(&dispatch_lb_kernel<32, true, kFp8Groups>)};
    size_t static_max = 0;
    for (const void *k : kernels) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, k);
        if (e != cudaSuccess) return e;
        static_max = fa.sharedSizeBytes > static_max ? fa.sharedSizeBytes : static_max;
    }
    const int limit = optin - (int)up(static_max, 128);
    for (const void *k : kernels) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
        if (e != cudaSuccess) return e;
    }
    __atomic_store_n(&g_smem_limit[dev], limit, __ATOMIC_RELEASE);
    return cudaSuccess;
}

cudaError_t launch_layout_counts(const LbParams &p, cudaStream_t s) {
    const size_t smem = sizeof(int32_t) * ((size_t)(p.E + p.R) + p.E + 1);
    layout_counts_kernel<<<p.nsuper, kLayoutThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_lb(const LbParams &p_in, bool fp8, int num_sms, cudaStream_t s) {
    LbParams p = p_in;
    const bool v32 = !fp8 && p.H % 16 == 0 &&
                     ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    const int VB = v32 ? 32 : 16;
    p.vec32 = (reinterpret_cast<uintptr_t>(p.recv) & 31) == 0;
    if (reinterpret_cast<uintptr_t>(p.pos) & 15) return cudaErrorInvalidValue;   // the handle's: 256-byte aligned
    if (!lb_unit_shape(p.H, fp8, VB, &p.splits, &p.chunk_bytes)) return cudaErrorInvalidValue;
    if ((int64_t)p.T * p.splits >= (int64_t(1) << 28)) return cudaErrorInvalidValue;   // stage tags hold 28 bits
    p.dyn_batch = p.splits * (fp8 ? EP_LB_DYN_TOKENS_FP8 : EP_LB_DYN_TOKENS_BF16);
    if (p.dyn_batch < 1) return cudaErrorInvalidValue;
    const size_t limit = smem_limit();
    const size_t fixed = carve(0, p.chunk_bytes, p.E).total;
    int ns = (int)(EP_LB_RING_BYTES / p.chunk_bytes);
    while (ns > 0 && carve(ns, p.chunk_bytes, p.E).total > limit) --ns;
    ns = ns > kMaxStages ? kMaxStages : ns;
    if (ns < 2 || fixed > limit) return cudaErrorInvalidValue;
    p.stages = ns;
    const size_t smem = carve(ns, p.chunk_bytes, p.E).total;
    const int grid = p.nchunks < num_sms ? p.nchunks : num_sms;
    if (grid <= 0) return cudaSuccess;
    if (fp8)
        return launch_pdl_lb(dispatch_lb_kernel<32, true, kFp8Groups>, grid, Shape<kFp8Groups>::kThreads, smem, s, p);
    return v32 ? launch_pdl_lb(dispatch_lb_kernel<32, false, 1>, grid, Shape<1>::kThreads, smem, s, p)
               : launch_pdl_lb(dispatch_lb_kernel<16, false, 1>, grid, Shape<1>::kThreads, smem, s, p);
}

}  // namespace ep
