// dispatch.cu -- token-major dispatch gather (bf16 copy, or fused FP8 E4M3
// quantisation) into the expert-contiguous received buffer (sm_100a).
//
// Each token row of x is read from HBM once and written to its K received
// rows (do_expand: one row per (token, expert) pair, EPBuffer.dispatch,
// bowenzhou.top "deepep/01-overview" section 1.1).  Padding rows that round
// each expert segment up to expert_alignment are zero-filled
// (do_zero_padding, same section).  FP8 follows the per-block scaling of
// "m.nlpx.cn/news/135159" section 4.1 and the quantise-before-send /
// restore-after-receive scheme of "2kiu.com/news/5702702" section 2.3, with
// one fp32 scale per 1x128 block of a token row.
//
// Work is split into units of similar byte volume, walked by a persistent
// grid: units [0, T*splits) copy one column range of one token to its K
// rows; units after that zero-fill the padding among kZeroRowsPerUnit
// consecutive received rows (only when expert_alignment > 1).  Copies use
// 32-byte (sm_100 256-bit) vector loads and stores when rows and pointers
// allow, else 16-byte ones; a bulk-copy (TMA engine) variant measured no
// faster on this write-bound pattern.

#include "ep_internal.cuh"
#include "fp8_block.cuh"

namespace ep {

namespace {

constexpr int kThreads = 256;

#ifndef EP_PDL_PREFETCH
#define EP_PDL_PREFETCH 1    // the staged kernel's L2 prefetch of x runs before its dependency wait,
                             // overlapping the layout (layout + dispatch 104.7 -> 101.9 us at the
                             // DeepSeek-V3 shape); 0: after it
#endif
#ifndef EP_FP8_PIPE
#define EP_FP8_PIPE 1        // the FP8 register kernel requests the next token's row before storing this
                             // one's codes (skew 94.6 -> 88.0 us, large 270.8 -> 260.8 us in one run)
#endif
#ifndef EP_FP8_MINB
#define EP_FP8_MINB 4        // resident blocks per SM the FP8 register kernel is compiled for (the
                             // pipelined loop at 3 blocks measured slower than without it)
#endif
#ifndef EP_LSU_UNROLL
#define EP_LSU_UNROLL 1      // vectors loaded per thread before its K stores (LSU bf16 path)
#endif
#ifndef EP_LSU_MINB
#define EP_LSU_MINB 8        // resident blocks per SM the LSU bf16 kernel is compiled for
#endif
constexpr int kUnroll = EP_LSU_UNROLL;

// ---------------------------------------------------------------------------
// LSU path: each thread moves VB-byte vectors (16, or 32 with sm_100 256-bit
// accesses when rows and pointers allow it).
// ---------------------------------------------------------------------------
template <int VB>
struct Vec;
template <>
struct Vec<16> {
    using T = uint4;
    static __device__ __forceinline__ T load(const void *p) { return ld_stream_v4(p); }
    static __device__ __forceinline__ void store(void *p, const T &v) { st_v4(p, v); }
    static __device__ __forceinline__ void store(void *p, const T &v, uint64_t pol) { st_v4_policy(p, v, pol); }
    static __device__ __forceinline__ T zero() { return make_uint4(0, 0, 0, 0); }
};
template <>
struct Vec<32> {
    using T = u32x8;
    static __device__ __forceinline__ T load(const void *p) { return ld_stream_v8(p); }
    static __device__ __forceinline__ void store(void *p, const T &v) { st_v8(p, v); }
    static __device__ __forceinline__ void store(void *p, const T &v, uint64_t pol) { st_v8_policy(p, v, pol); }
    static __device__ __forceinline__ T zero() {
        T z;
#pragma unroll
        for (int i = 0; i < 8; ++i) z.v[i] = 0;
        return z;
    }
};

// Zero-fill unit z: padding rows among received rows [z*8, z*8+8).
template <int VB>
__device__ __forceinline__ void zero_fill_unit(const DispatchParams &p, int z, int rows, int row_bytes,
                                               int tid, int nthreads) {
    using V = Vec<VB>;
    const int nv = row_bytes / VB;
    const int r0 = z * kZeroRowsPerUnit, r1 = min(rows, r0 + kZeroRowsPerUnit);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    for (int r = r0; r < r1; ++r) {
        if (__ldg(&p.row_src[r]) >= 0) continue;
        uint8_t *o = recv + (int64_t)r * row_bytes;
        for (int v = tid; v < nv; v += nthreads) V::store(o + (int64_t)v * VB, V::zero());
    }
}

// ---------------------------------------------------------------------------
// Low-latency static layout (lesson14_deepep section 2(1): decode buffers are
// pre-allocated per expert and the per-expert count is the mask).  Expert e
// owns rows e*M .. e*M+M-1, filled in (token, k) order, so the slot of pair
// (t, k) is the number of earlier pairs with the same expert.  Every CTA
// walks its tokens in increasing order and keeps a shared-memory histogram
// of the pairs of all tokens before the current one (each CTA re-reads the
// ids it has not counted yet: T*K ids at most, an L2 hit), so no CTA waits
// on another and layout and copy are one launch.  The grid's last CTA only
// counts all pairs and writes recv_count.
// ---------------------------------------------------------------------------
struct LlState {
    int32_t *hist;   // [E] pairs per expert among tokens [0, upto)
    int32_t *ids;    // [kMaxTopk] this token's ids (-1 masked, -2 invalid)
    int upto;
};

__device__ __forceinline__ void ll_init(const DispatchParams &p, LlState &st) {
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) st.hist[e] = 0;
    st.upto = 0;
    __syncthreads();
}

__device__ __forceinline__ void ll_advance(const DispatchParams &p, LlState &st, int t) {
    for (int64_t i = (int64_t)st.upto * p.K + threadIdx.x; i < (int64_t)t * p.K; i += blockDim.x) {
        const int64_t e = __ldg(&p.topk_idx[i]);
        if (e >= 0 && e < p.E) atomicAdd(&st.hist[e], 1);
    }
    st.upto = t;
}

// Destinations of token t's K pairs into s_dst (split 0 also writes pos);
// ends with a block barrier.
__device__ __forceinline__ void ll_destinations(const DispatchParams &p, LlState &st, int t, bool write_pos,
                                                int32_t *s_dst) {
    if (t > st.upto) ll_advance(p, st, t);
    if (threadIdx.x < p.K) {
        const int64_t e = __ldg(&p.topk_idx[(int64_t)t * p.K + threadIdx.x]);
        st.ids[threadIdx.x] = (e >= 0 && e < p.E) ? (int)e : (e == -1 ? -1 : -2);
    }
    __syncthreads();
    if (threadIdx.x < p.K) {
        const int k = threadIdx.x, e = st.ids[k];
        int dst = -1;
        if (e >= 0) {
            int slot = st.hist[e];
            for (int j = 0; j < k; ++j) slot += st.ids[j] == e;
            if (slot < p.ll_M)
                dst = e * p.ll_M + slot;
            else if (write_pos)
                atomicOr(p.status, EP_DEV_SLOT_OVERFLOW);
        } else if (e == -2 && write_pos) {
            atomicOr(p.status, EP_DEV_BAD_EXPERT);
        }
        s_dst[k] = dst;
        if (write_pos) p.pos_out[(int64_t)t * p.K + k] = dst;
    }
    __syncthreads();
}

// The count CTA: recv_count[e] = min(pairs of expert e, M).
__device__ __forceinline__ void ll_count(const DispatchParams &p, LlState &st) {
    ll_advance(p, st, p.T);
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) p.recv_count[e] = min(st.hist[e], p.ll_M);
}

template <int VB, bool LL>
__global__ void __launch_bounds__(kThreads, EP_LSU_MINB) dispatch_bf16_kernel(DispatchParams p) {
    using V = Vec<VB>;
    using VT = typename V::T;
    __shared__ int32_t s_dst[kMaxTopk];
    const int row_bytes = p.H * 2;
    const int nv = row_bytes / VB;
    const int vps = (nv + p.splits - 1) / p.splits;
    const int total = p.n_token_units + p.n_zero_units;
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    int rows = -1;
    LlState st;
    int nblk = gridDim.x;
    pdl_wait();   // the layout (or whatever ran before) is complete and visible
    if constexpr (LL) {
        extern __shared__ int32_t ll_smem[];
        st.ids = ll_smem;
        st.hist = ll_smem + kMaxTopk;
        ll_init(p, st);
        if (p.recv_count) {
            nblk = gridDim.x - 1;
            if (blockIdx.x == nblk) {
                ll_count(p, st);
                return;
            }
        }
    }
    for (int u = blockIdx.x; u < total; u += nblk) {
        if (u < p.n_token_units) {
            const int t = u / p.splits, s = u - t * p.splits;
            const int v0 = s * vps, v1 = min(nv, v0 + vps);
            const uint8_t *xr = x + (int64_t)t * row_bytes;
            // the first vectors of the row are loaded before the destinations
            // are known, so the two memory round trips overlap
            VT buf[kUnroll];
            const int vfirst = v0 + threadIdx.x;
#pragma unroll
            for (int j = 0; j < kUnroll; ++j)
                if (vfirst + j * kThreads < v1) buf[j] = V::load(xr + (int64_t)(vfirst + j * kThreads) * VB);
            if constexpr (LL) {
                ll_destinations(p, st, t, s == 0, s_dst);
            } else {
                if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
                __syncthreads();
            }
            for (int v = vfirst; v < v1; v += kThreads * kUnroll) {
                if (v != vfirst) {
#pragma unroll
                    for (int j = 0; j < kUnroll; ++j)
                        if (v + j * kThreads < v1) buf[j] = V::load(xr + (int64_t)(v + j * kThreads) * VB);
                }
                for (int k = 0; k < p.K; ++k) {
                    const int dst = s_dst[k];
                    if (dst < 0) continue;
                    uint8_t *o = recv + (int64_t)dst * row_bytes;
#pragma unroll
                    for (int j = 0; j < kUnroll; ++j)
                        if (v + j * kThreads < v1) V::store(o + (int64_t)(v + j * kThreads) * VB, buf[j]);
                }
            }
            __syncthreads();
        } else {
            if (rows < 0) rows = __ldg(&p.eoff[p.E]);
            zero_fill_unit<VB>(p, u - p.n_token_units, rows, row_bytes, threadIdx.x, kThreads);
        }
    }
}

// ---------------------------------------------------------------------------
// Staged path (bf16): a producer warp streams row chunks of x into a ring of
// shared-memory stages with bulk global->shared copies (TMA engine; each
// stage's "full" mbarrier counts the bytes in).  Consumer groups of 7 warps
// take every kStagedGroups-th unit: a group waits for its stage, reads each
// vector of it once and stores it to the unit's K received rows, then
// releases the stage on its "empty" mbarrier.  Loads run ahead of the
// stores, and several groups keep enough stores in flight per SM to cover
// HBM write latency.  Every wait is bounded; a timeout sets
// EP_DEV_WAIT_TIMEOUT.
// ---------------------------------------------------------------------------
#ifndef EP_DISPATCH_STAGED
#define EP_DISPATCH_STAGED 1
#endif
#ifndef EP_STAGED_CHUNK_MAX
#define EP_STAGED_CHUNK_MAX 8192    // bytes of a row per unit (rows split into chunks)
#endif
#ifndef EP_STAGED_SMEM
#define EP_STAGED_SMEM (112 * 1024) // shared-memory ring budget per CTA
#endif
#ifndef EP_STAGED_PREFETCH
#define EP_STAGED_PREFETCH 1        // 0: none, 1: L2 prefetch of the CTA's x rows (evict_last), 2: evict_normal
#endif
#ifndef EP_STAGED_STORE_EVICT_FIRST
#define EP_STAGED_STORE_EVICT_FIRST 1
#endif
#ifndef EP_STAGED_GROUPS
#define EP_STAGED_GROUPS 1          // consumer groups working on different stages at once
#endif
constexpr int kGroupWarps = 7;                     // warps per consumer group
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kStagedGroups = EP_STAGED_GROUPS;
// warp 0 produces, then kStagedGroups consumer groups, then one zero-fill warp
constexpr int kStagedThreads = 32 + kStagedGroups * kGroupThreads + 32;
constexpr int kZeroWarp = (kStagedThreads / 32) - 1;
constexpr int kZeroSmemBytes = 8192;   // zeroed shared memory the zero-fill warp copies from
constexpr int kStagedMaxStages = 16;
constexpr int kStagedPosInts = 4096;  // staged pos entries (units x K) per window

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ __forceinline__ size_t staged_smem_bytes(int stages, int chunk) {
    return align_up((size_t)stages * chunk, 128) + 2 * kStagedMaxStages * sizeof(uint64_t) +
           kStagedPosInts * sizeof(int32_t) + kZeroSmemBytes;
}

// The zero-fill warp: lane l takes zero units blockIdx.x + (l + 32 i) * gridDim.x
// and writes every padding row among them with bulk shared->global copies
// from a zeroed shared-memory block (the TMA engine does the writing, so no
// consumer thread is spent on it).
__device__ __forceinline__ void zero_fill_warp(const DispatchParams &p, int rows, int row_bytes,
                                               const uint8_t *zeros, int lane) {
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    for (int z = blockIdx.x + lane * gridDim.x; z < p.n_zero_units; z += 32 * gridDim.x) {
        const int r0 = z * kZeroRowsPerUnit, r1 = min(rows, r0 + kZeroRowsPerUnit);
        for (int r = r0; r < r1; ++r) {
            if (__ldg(&p.row_src[r]) >= 0) continue;
            uint8_t *o = recv + (int64_t)r * row_bytes;
            for (int off = 0; off < row_bytes; off += kZeroSmemBytes)
                bulk_s2g(o + off, zeros, (uint32_t)min(kZeroSmemBytes, row_bytes - off));
        }
        bulk_commit();
    }
    bulk_wait_all();
}

template <int VB>
__device__ __forceinline__ typename Vec<VB>::T lds_vec(const uint8_t *p);
template <>
__device__ __forceinline__ uint4 lds_vec<16>(const uint8_t *p) {
    return *reinterpret_cast<const uint4 *>(p);
}
template <>
__device__ __forceinline__ u32x8 lds_vec<32>(const uint8_t *p) {
    const uint4 a = *reinterpret_cast<const uint4 *>(p), b = *reinterpret_cast<const uint4 *>(p + 16);
    u32x8 r;
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
    return r;
}

template <int VB>
__global__ void __launch_bounds__(kStagedThreads, 1) dispatch_bf16_staged_kernel(DispatchParams p) {
    static_assert(kStagedThreads <= 1024, "too many consumer groups");
    using V = Vec<VB>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int NS = p.stages;
    const int row_bytes = p.H * 2;
    const int chunk = row_bytes / p.splits;
    uint8_t *buf = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + align_up((size_t)NS * chunk, 128));
    uint64_t *empty = full + kStagedMaxStages;
    int32_t *s_pos = reinterpret_cast<int32_t *>(empty + kStagedMaxStages);
    uint8_t *zeros = reinterpret_cast<uint8_t *>(s_pos + kStagedPosInts);
    __shared__ int s_abort;
    __shared__ int s_rows;
    volatile int *abort_flag = &s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_cta = p.n_token_units > (int)blockIdx.x
                          ? (p.n_token_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                          : 0;
    const int win = max(1, kStagedPosInts / p.K);
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);

    if (p.n_zero_units) {
        for (int i = threadIdx.x; i < kZeroSmemBytes / 16; i += kStagedThreads)
            reinterpret_cast<uint4 *>(zeros)[i] = make_uint4(0, 0, 0, 0);
        fence_async_smem();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kGroupWarps);
        }
        fence_async_smem();
        s_abort = 0;
    }
#if EP_PDL_PREFETCH && EP_STAGED_PREFETCH
    // an L2 prefetch may run before the wait: L2 is where writes land, so a
    // line prefetched while the previous kernel still writes it is updated there
    if (p.prefetch_x && threadIdx.x == 0) {
        const uint64_t pol_x = policy_evict_last();
        for (int i = 0; i < n_cta; ++i) {
            const int u = blockIdx.x + i * gridDim.x;
            const int t = u / p.splits, part = u - t * p.splits;
            bulk_prefetch_l2(x + (int64_t)t * row_bytes + (int64_t)part * chunk, chunk, pol_x);
        }
    }
#endif
    pdl_wait();   // shared-memory set-up overlapped the previous kernel; global reads start here
    if (threadIdx.x == 0) s_rows = p.n_zero_units ? __ldg(&p.eoff[p.E]) : 0;
    __syncthreads();

#if EP_STAGED_PREFETCH && !EP_PDL_PREFETCH
    // bring all of this CTA's x chunks into L2 up front: HBM serves a short
    // burst of reads, then only the stream of received-row writes, and the
    // chunks stay in L2 (evict_last) while that stream passes through
    if (p.prefetch_x && threadIdx.x == 0) {
#if EP_STAGED_PREFETCH == 1
        const uint64_t pol_x = policy_evict_last();
#else
        uint64_t pol_x;
        asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol_x));
#endif
        for (int i = 0; i < n_cta; ++i) {
            const int u = blockIdx.x + i * gridDim.x;
            const int t = u / p.splits, part = u - t * p.splits;
            bulk_prefetch_l2(x + (int64_t)t * row_bytes + (int64_t)part * chunk, chunk, pol_x);
        }
    }
#endif
#if EP_STAGED_STORE_EVICT_FIRST
    const uint64_t pol_out = policy_evict_first();
#endif

    int issued = 0;   // producer: units whose load was issued
    for (int w0 = 0; w0 < n_cta; w0 += win) {
        const int wn = min(win, n_cta - w0);
        for (int i = threadIdx.x; i < wn * p.K; i += kStagedThreads) {
            const int u = blockIdx.x + (w0 + i / p.K) * gridDim.x;
            s_pos[i] = __ldg(&p.pos[(int64_t)(u / p.splits) * p.K + (i % p.K)]);
        }
        __syncthreads();
        if (warp == 0) {
            if (lane == 0) {
                for (int i = w0; i < w0 + wn && !*abort_flag; ++i) {
                    const int s = i % NS, use = i / NS;
                    if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1, p.wait_limit_ns)) {
                        atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    const int u = blockIdx.x + i * gridDim.x;
                    const int t = u / p.splits, part = u - t * p.splits;
                    mbar_arrive_expect_tx(&full[s], chunk);
                    bulk_g2s(buf + (size_t)s * chunk, x + (int64_t)t * row_bytes + (int64_t)part * chunk, chunk,
                             &full[s]);
                    ++issued;
                }
            }
        } else if (warp == kZeroWarp) {
            if (w0 == 0) zero_fill_warp(p, s_rows, row_bytes, zeros, lane);
        } else {
            const int grp = (threadIdx.x - 32) / kGroupThreads;
            const int gtid = (threadIdx.x - 32) - grp * kGroupThreads;
            const int nv = chunk / VB;
            for (int i = w0 + ((grp - w0 % kStagedGroups + kStagedGroups) % kStagedGroups); i < w0 + wn;
                 i += kStagedGroups) {
                const int s = i % NS;
                if (!mbar_wait_bounded(&full[s], (i / NS) & 1, p.wait_limit_ns)) {
                    atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                const int part = (blockIdx.x + i * gridDim.x) % p.splits;
                const uint8_t *src = buf + (size_t)s * chunk;
                const int32_t *dsts = s_pos + (i - w0) * p.K;
                for (int v = gtid; v < nv; v += kGroupThreads) {
                    const typename V::T val = lds_vec<VB>(src + v * VB);
                    for (int k = 0; k < p.K; ++k) {
                        const int dst = dsts[k];
                        if (dst >= 0)
#if EP_STAGED_STORE_EVICT_FIRST
                            V::store(recv + (int64_t)dst * row_bytes + (int64_t)part * chunk + (int64_t)v * VB, val,
                                     pol_out);
#else
                            V::store(recv + (int64_t)dst * row_bytes + (int64_t)part * chunk + (int64_t)v * VB, val);
#endif
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
        }
        __syncthreads();
        if (*abort_flag) break;
    }
    if (n_cta == 0 && warp == kZeroWarp) zero_fill_warp(p, s_rows, row_bytes, zeros, lane);
    if (*abort_flag && threadIdx.x == 0) {
        // let every issued load land before the CTA's shared memory goes away
        for (int j = max(0, issued - NS); j < issued; ++j)
            mbar_wait_bounded(&full[j % NS], (j / NS) & 1, p.wait_limit_ns);
    }
}

// Index of the scale of received row `row`, block b, in either layout.
// Column-major scales come in groups of scale_group_rows rows (the whole
// buffer, or one expert's M slots), each group [H/128][scale_ld].
__device__ __forceinline__ int64_t scale_index(const DispatchParams &p, int row, int b, int NB) {
    if (p.scale_ld == 0) return (int64_t)row * NB + b;
    const int g = row / p.scale_group_rows;
    return ((int64_t)g * NB + b) * p.scale_ld + (row - g * p.scale_group_rows);
}

// EPT bf16 elements per thread (16: 16-byte accesses, 32: 32-byte accesses);
// TPB = 128 / EPT consecutive lanes share one 1x128 block and reduce its
// amax with shuffles.  Each thread stores EPT code bytes per received row.
template <int EPT, bool LL>
__global__ void __launch_bounds__(kThreads, EP_FP8_MINB) dispatch_fp8_kernel(DispatchParams p) {
    constexpr int TPB = 128 / EPT;
    constexpr int NW = EPT / 2;              // bf16x2 words loaded per thread
    __shared__ int32_t s_dst[kMaxTopk];
    const int NB = p.H / 128;
    const int nthr_row = p.H / EPT;
    const int total = p.n_token_units + p.n_zero_units;
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    int rows = -1;
    LlState st;
    int nblk = gridDim.x;
    if constexpr (!LL) {
        // this CTA's token rows into L2 (evict_last) before the dependency
        // wait, as in the staged bf16 kernel: L2 is where writes land, so a
        // line prefetched while the previous kernel still writes it is updated
        if (p.prefetch_x && threadIdx.x == 0) {
            const uint64_t pol_x = policy_evict_last();
            for (int t = blockIdx.x; t < p.n_token_units; t += gridDim.x)
                bulk_prefetch_l2(x + (int64_t)t * p.H * 2, (uint32_t)p.H * 2, pol_x);
        }
    }
    pdl_wait();   // the layout (or whatever ran before) is complete and visible
    if constexpr (LL) {
        extern __shared__ int32_t ll_smem[];
        st.ids = ll_smem;
        st.hist = ll_smem + kMaxTopk;
        ll_init(p, st);
        if (p.recv_count) {
            nblk = gridDim.x - 1;
            if (blockIdx.x == nblk) {
                ll_count(p, st);
                return;
            }
        }
    }
    int u = blockIdx.x;
#if EP_FP8_PIPE
    if (!LL && nthr_row <= kThreads) {
        // software-pipelined token loop: the next token's row is requested
        // before this token's codes are stored, so one row's loads are always
        // in flight behind the stores
        const bool act = threadIdx.x < nthr_row;
        unsigned int w[NW];
        if (act && u < p.n_token_units) {
            Fp8Io<EPT>::load(x + (int64_t)u * p.H * 2 + (int64_t)threadIdx.x * EPT * 2, w);
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = 0;
        }
        for (; u < p.n_token_units; u += nblk) {
            if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)u * p.K + threadIdx.x]);
            __syncthreads();
            const int un = u + nblk;
            unsigned int wn[NW];
            if (act && un < p.n_token_units) {
                Fp8Io<EPT>::load(x + (int64_t)un * p.H * 2 + (int64_t)threadIdx.x * EPT * 2, wn);
            } else {
#pragma unroll
                for (int i = 0; i < NW; ++i) wn[i] = 0;
            }
            unsigned int q[8];
            const float scale = quantize_block<TPB, NW>(w, q);
            if (act) {
                const int b = threadIdx.x / TPB;
                const bool lead = (threadIdx.x % TPB) == 0;
                for (int k = 0; k < p.K; ++k) {
                    const int dst = s_dst[k];
                    if (dst < 0) continue;
                    Fp8Io<EPT>::store(recv + (int64_t)dst * p.H + (int64_t)threadIdx.x * EPT, q);
                    if (lead) p.recv_scale[scale_index(p, dst, b, NB)] = scale;
                }
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = wn[i];
        }
    }
#endif
    for (; u < total; u += nblk) {
        if (u < p.n_token_units) {
            const int t = u;
            const uint8_t *xr = x + (int64_t)t * p.H * 2;
            // the first part of the row is loaded before the destinations are
            // known, so the two memory round trips overlap
            unsigned int w[NW];
            if (threadIdx.x < nthr_row) {
                Fp8Io<EPT>::load(xr + (int64_t)threadIdx.x * EPT * 2, w);
            } else {
#pragma unroll
                for (int i = 0; i < NW; ++i) w[i] = 0;
            }
            if constexpr (LL) {
                ll_destinations(p, st, t, true, s_dst);
            } else {
                if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
                __syncthreads();
            }
            for (int g0 = 0; g0 < nthr_row; g0 += kThreads) {
                const int g = g0 + threadIdx.x;
                const bool act = g < nthr_row;
                if (g0 > 0) {
                    if (act) {
                        Fp8Io<EPT>::load(xr + (int64_t)g * EPT * 2, w);
                    } else {
#pragma unroll
                        for (int i = 0; i < NW; ++i) w[i] = 0;
                    }
                }
                unsigned int q[8];
                const float scale = quantize_block<TPB, NW>(w, q);
                if (act) {
                    const int b = g / TPB;
                    const bool lead = (g % TPB) == 0;
                    for (int k = 0; k < p.K; ++k) {
                        const int dst = s_dst[k];
                        if (dst < 0) continue;
                        Fp8Io<EPT>::store(recv + (int64_t)dst * p.H + (int64_t)g * EPT, q);
                        if (lead) p.recv_scale[scale_index(p, dst, b, NB)] = scale;
                    }
                }
            }
            __syncthreads();
        } else {
            if (rows < 0) rows = __ldg(&p.eoff[p.E]);
            const int r0 = (u - p.n_token_units) * kZeroRowsPerUnit;
            const int r1 = min(rows, r0 + kZeroRowsPerUnit);
            for (int r = r0; r < r1; ++r) {
                if (__ldg(&p.row_src[r]) >= 0) continue;
                uint8_t *o = recv + (int64_t)r * p.H;
                for (int v = threadIdx.x; v < p.H / 16; v += kThreads) st_v4(o + v * 16, make_uint4(0, 0, 0, 0));
                for (int b = threadIdx.x; b < NB; b += kThreads) p.recv_scale[scale_index(p, r, b, NB)] = 0.0f;
            }
        }
    }
}

}  // namespace

// Staged launch shape for rows of row_bytes with VB-byte vectors: the row is
// split into the fewest power-of-two chunks of at most EP_STAGED_CHUNK_MAX
// bytes (a multiple of VB); 0 stages means "use the register kernel".
static void staged_shape(int row_bytes, int VB, int *splits, int *stages) {
    int sp = 1;
    while (sp <= 64 && (row_bytes / sp > EP_STAGED_CHUNK_MAX || row_bytes % (sp * VB) != 0)) sp *= 2;
    *splits = sp;
    *stages = 0;
    if (!EP_DISPATCH_STAGED || sp > 64 || row_bytes % (sp * VB) != 0) return;
    int ns = EP_STAGED_SMEM / (row_bytes / sp);
    ns = ns > kStagedMaxStages ? kStagedMaxStages : ns;
    if (ns >= 3) *stages = ns;
}

cudaError_t dispatch_prepare() {
    const int smem = (int)staged_smem_bytes(kStagedMaxStages, EP_STAGED_CHUNK_MAX);
    const void *kernels[] = {reinterpret_cast<const void *>(&dispatch_bf16_staged_kernel<32>),
                             reinterpret_cast<const void *>(&dispatch_bf16_staged_kernel<16>)};
    for (const void *k : kernels) {
        const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Launch that may start while the previous kernel on the stream finishes
// (programmatic stream serialization); the kernels wait with pdl_wait()
// before touching global memory.
template <typename Kernel>
static cudaError_t launch_pdl(Kernel kernel, int grid, int block, size_t smem, cudaStream_t s,
                              const DispatchParams &p) {
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

cudaError_t launch_dispatch_bf16(const DispatchParams &p_in, int num_sms, cudaStream_t s) {
    static OccupancyCache occ16, occ32;
    DispatchParams p = p_in;
    const bool v32 = (p.H % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    const int row_bytes = p.H * 2;
    int splits = 1, stages = 0;
    staged_shape(row_bytes, v32 ? 32 : 16, &splits, &stages);
    if (stages > 0 && p.T * splits >= 4 * num_sms) {
        p.splits = splits;
        p.stages = stages;
        p.n_token_units = p.T * splits;
        const int units = p.n_token_units + p.n_zero_units;
        const int grid = units < num_sms ? units : num_sms;
        const size_t smem = staged_smem_bytes(stages, row_bytes / splits);
        return v32 ? launch_pdl(dispatch_bf16_staged_kernel<32>, grid, kStagedThreads, smem, s, p)
                   : launch_pdl(dispatch_bf16_staged_kernel<16>, grid, kStagedThreads, smem, s, p);
    }
    const int units = p.n_token_units + p.n_zero_units;
    if (v32) {
        const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<32, false>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ32), num_sms);
        return launch_pdl(dispatch_bf16_kernel<32, false>, grid, kThreads, 0, s, p);
    } else {
        const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<16, false>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ16), num_sms);
        return launch_pdl(dispatch_bf16_kernel<16, false>, grid, kThreads, 0, s, p);
    }
}

// Low-latency launches: the register kernels with in-kernel destinations.
// The copy CTAs come from the occupancy-sized persistent grid; one more CTA
// counts all pairs into recv_count.
static size_t ll_smem_bytes(int E) { return sizeof(int32_t) * (size_t)(kMaxTopk + E); }

cudaError_t launch_ll_dispatch(const DispatchParams &p_in, bool fp8, int num_sms, cudaStream_t s) {
    static OccupancyCache occ[4];
    DispatchParams p = p_in;
    p.n_zero_units = 0;
    const size_t smem = ll_smem_bytes(p.E);
    const size_t smem_max = ll_smem_bytes(kMaxExperts);
    const bool v32 = (fp8 || p.H % 16 == 0) &&
                     ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    const void *k;
    OccupancyCache *slot;
    if (fp8) {
        p.splits = 1;
        k = v32 ? reinterpret_cast<const void *>(&dispatch_fp8_kernel<32, true>)
                : reinterpret_cast<const void *>(&dispatch_fp8_kernel<16, true>);
        slot = &occ[v32 ? 0 : 1];
    } else {
        // split rows so that a small batch still spreads over the SMs
        const int nv = p.H * 2 / (v32 ? 32 : 16);
        int sp = 1;
        while (sp < 8 && p.T * sp < 2 * num_sms && nv / (sp * 2) >= kThreads / 2) sp *= 2;
        p.splits = sp;
        k = v32 ? reinterpret_cast<const void *>(&dispatch_bf16_kernel<32, true>)
                : reinterpret_cast<const void *>(&dispatch_bf16_kernel<16, true>);
        slot = &occ[v32 ? 2 : 3];
    }
    p.n_token_units = p.T * p.splits;
    const int grid = persistent_grid(p.n_token_units, blocks_per_sm(k, kThreads, smem_max, slot), num_sms) +
                     (p.recv_count ? 1 : 0);
    // programmatic stream serialization, as for the normal dispatch: the
    // kernels wait (pdl_wait) before their first global read
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    void *args[] = {&p};
    return cudaLaunchKernelExC(&cfg, k, args);
}

// FP8 uses the register kernel: quantising from a staged ring with one
// consumer group per SM measured slower (the quantisation needs the
// register kernel's four resident blocks per SM).
cudaError_t launch_dispatch_fp8(const DispatchParams &p, int num_sms, cudaStream_t s) {
    static OccupancyCache occ16, occ32;
    const int units = p.n_token_units + p.n_zero_units;
    const bool v32 = ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    if (v32) {
        const void *k = reinterpret_cast<const void *>(&dispatch_fp8_kernel<32, false>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ32), num_sms);
        return launch_pdl(dispatch_fp8_kernel<32, false>, grid, kThreads, 0, s, p);
    } else {
        const void *k = reinterpret_cast<const void *>(&dispatch_fp8_kernel<16, false>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ16), num_sms);
        return launch_pdl(dispatch_fp8_kernel<16, false>, grid, kThreads, 0, s, p);
    }
}

}  // namespace ep
