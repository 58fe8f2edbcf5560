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
// These are the register kernels: ep_dispatch / ep_dispatch_fp8 use them for
// batches too small to fill the GPU (fewer than two tokens per SM), and the
// low-latency layout uses them always; larger batches go to the chunked
// kernel of dispatch_lb.cu.  Work is split into units of similar byte
// volume, walked by a persistent grid: units [0, T*splits) copy one column
// range of one token to its K rows; units after that zero-fill the padding
// among kZeroRowsPerUnit consecutive received rows (only when
// expert_alignment > 1).  Copies use 32-byte (sm_100 256-bit) vector loads
// and stores when rows and pointers allow, else 16-byte ones.

#include "ep_internal.cuh"
#include "fp8_block.cuh"

namespace ep {

namespace {

constexpr int kThreads = 256;

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
        // wait: L2 is where writes land, so a line prefetched while the
        // previous kernel still writes it is updated
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

// ---------------------------------------------------------------------------
// Layout and dispatch in one launch, for batches too small to fill the GPU
// (ep_layout_dispatch with fewer than two tokens per SM).  The padded layout
// of a small batch is cheap enough to compute in every CTA: each CTA reads
// all T*K ids (an L2 hit after the first), counts every expert and the pairs
// of the tokens before its own, and scans the padded counts into the expert
// offsets.  A pair's row is then its expert's offset + the pairs of that
// expert in earlier tokens + the earlier slots of its own token with the same
// expert: the (token, k) order of the lesson14_deepep practice task's queues.
// CTA c handles tokens c, c + G, ...: it writes their routing entries, their
// is_token_in_rank rows and their copies (the first row is loaded before the
// counting, so the two overlap); the padding rows of experts c, c + G, ...
// are written as well; CTA 0 writes the counts and offsets, the last CTA the
// distinct tokens per rank.  No CTA waits on another.  With p.x == nullptr
// the same kernel computes the layout alone (ep_get_layout of a small batch).
// ---------------------------------------------------------------------------
template <bool FP8, int W>   // W: bf16 elements per thread (FP8) or vector bytes (bf16)
__device__ __forceinline__ void small_layout_dispatch(const DispatchParams &p, const LayoutParams &lp) {
    __shared__ int32_t s_tot[kMaxExperts + 1];   // pairs per expert (later: tokens per rank, last CTA)
    __shared__ int32_t s_before[kMaxExperts];    // pairs per expert among tokens [0, upto)
    __shared__ int32_t s_eoff[kMaxExperts + 1];  // padded expert offsets
    __shared__ int32_t s_dst[kMaxTopk];
    __shared__ int32_t s_id[kMaxTopk];          // the current token's ids (-1: none or invalid)
    __shared__ int16_t s_rk[kMaxExperts];        // rank of expert e (e / L)
    __shared__ int32_t s_warp[kThreads / 32 + 1];
    constexpr int EPT = W, TPB = 128 / (FP8 ? W : 128), NW = W / 2;
    const int E = lp.E, K = lp.K, T = lp.T, R = lp.R, L = lp.L, A = lp.A, H = p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, G = gridDim.x;
    const int64_t *idx = lp.topk_idx;
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    const int row_bytes = FP8 ? H : H * 2;
    const bool copy = x != nullptr;   // false: the layout alone (ep_get_layout of a small batch)
    pdl_launch_dependents();          // a kernel launched next may start its set-up now

    // the first token's row is requested before the counting
    unsigned int w8[FP8 ? NW : 1];
    typename Vec<FP8 ? 16 : W>::T v0;
    const int nthr_row = FP8 ? H / EPT : row_bytes / W;
    if (copy && blockIdx.x < T && tid < nthr_row) {
        if constexpr (FP8)
            Fp8Io<EPT>::load(x + (int64_t)blockIdx.x * H * 2 + (int64_t)tid * EPT * 2, w8);
        else
            v0 = Vec<W>::load(x + (int64_t)blockIdx.x * row_bytes + (int64_t)tid * W);
    }

    for (int e = tid; e < E; e += kThreads) {
        s_tot[e] = 0;
        s_before[e] = 0;
        s_rk[e] = (int16_t)(e / L);
    }
    __syncthreads();
    const int64_t npairs = (int64_t)T * K, nbefore = (int64_t)blockIdx.x * K;
    bool bad = false;
    for (int64_t i = tid; i < npairs; i += kThreads) {
        const int64_t e = __ldg(idx + i);
        if (e >= 0 && e < E) {
            atomicAdd(&s_tot[e], 1);
            if (i < nbefore) atomicAdd(&s_before[e], 1);
        } else if (e != -1) {
            bad = true;
        }
    }
    if (bad && blockIdx.x == 0) atomicOr(lp.status, EP_DEV_BAD_EXPERT);
    __syncthreads();
    // padded exclusive offsets: per = E / kThreads consecutive experts per thread
    {
        const int per = (E + kThreads - 1) / kThreads;
        const int lo = min(E, tid * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) sum += (s_tot[e] + A - 1) / A * A;
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) s_warp[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            const int wv = lane < kThreads / 32 ? s_warp[lane] : 0;
            int wi = wv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += v;
            }
            if (lane < kThreads / 32) s_warp[lane] = wi - wv;
            if (lane == kThreads / 32 - 1) s_warp[kThreads / 32] = wi;
        }
        __syncthreads();
        int run = s_warp[warp] + inc - sum;
        for (int e = lo; e < hi; ++e) {
            s_eoff[e] = run;
            run += (s_tot[e] + A - 1) / A * A;
        }
        if (tid == 0) s_eoff[E] = s_warp[kThreads / 32];
    }
    __syncthreads();

    const int NB = H / 128;
    int upto = blockIdx.x;
    for (int t = blockIdx.x; t < T; t += G) {
        if (t > upto) {   // pairs of the tokens between this CTA's previous token and t
            for (int64_t i = (int64_t)upto * K + tid; i < (int64_t)t * K; i += kThreads) {
                const int64_t e = __ldg(idx + i);
                if (e >= 0 && e < E) atomicAdd(&s_before[e], 1);
            }
            upto = t;
            __syncthreads();
            if (copy && tid < nthr_row) {   // this token's row (the first one was loaded before the counting)
                if constexpr (FP8)
                    Fp8Io<EPT>::load(x + (int64_t)t * H * 2 + (int64_t)tid * EPT * 2, w8);
                else
                    v0 = Vec<W>::load(x + (int64_t)t * row_bytes + (int64_t)tid * W);
            }
        }
        const int64_t *row = idx + (int64_t)t * K;
        if (tid < K) {
            const int64_t e = __ldg(row + tid);
            s_id[tid] = (e >= 0 && e < E) ? (int)e : -1;
        }
        __syncthreads();
        if (tid < K) {
            const int e = s_id[tid];
            int dst = -1;
            if (e >= 0) {
                int same = 0;
                for (int k2 = 0; k2 < tid; ++k2) same += s_id[k2] == e;
                dst = s_eoff[e] + s_before[e] + same;
                lp.row_src[dst] = t;
                lp.row_slot[dst] = tid;
                if (lp.topk_weights) lp.row_weight[dst] = __ldg(lp.topk_weights + (int64_t)t * K + tid);
            }
            lp.pos[(int64_t)t * K + tid] = dst;
            s_dst[tid] = dst;
        }
        if (lp.u_in_rank) {
            for (int r = tid; r < R; r += kThreads) {
                uint8_t in = 0;
                for (int k = 0; k < K; ++k) {
                    const int e = s_id[k];
                    if (e >= 0 && s_rk[e] == r) in = 1;
                }
                lp.u_in_rank[(int64_t)t * R + r] = in;
            }
        }
        __syncthreads();
        if (!copy) continue;
        if constexpr (FP8) {
            const uint8_t *xr = x + (int64_t)t * H * 2;
            for (int g0 = 0; g0 < nthr_row; g0 += kThreads) {
                const int g = g0 + tid;
                const bool act = g < nthr_row;
                if (g0 > 0) {
                    if (act) {
                        Fp8Io<EPT>::load(xr + (int64_t)g * EPT * 2, w8);
                    } else {
#pragma unroll
                        for (int i = 0; i < NW; ++i) w8[i] = 0;
                    }
                } else if (!act) {
#pragma unroll
                    for (int i = 0; i < NW; ++i) w8[i] = 0;
                }
                unsigned int q[8];
                const float scale = quantize_block<TPB, NW>(w8, q);
                if (act) {
                    const int b = g / TPB;
                    const bool lead = (g % TPB) == 0;
                    for (int k = 0; k < K; ++k) {
                        const int dst = s_dst[k];
                        if (dst < 0) continue;
                        Fp8Io<EPT>::store(recv + (int64_t)dst * H + (int64_t)g * EPT, q);
                        if (lead) p.recv_scale[scale_index(p, dst, b, NB)] = scale;
                    }
                }
            }
        } else {
            const uint8_t *xr = x + (int64_t)t * row_bytes;
            for (int v = tid; v < nthr_row; v += kThreads) {
                const typename Vec<W>::T val = v == tid ? v0 : Vec<W>::load(xr + (int64_t)v * W);
                for (int k = 0; k < K; ++k) {
                    const int dst = s_dst[k];
                    if (dst >= 0) Vec<W>::store(recv + (int64_t)dst * row_bytes + (int64_t)v * W, val);
                }
            }
        }
        __syncthreads();
    }

    // padding rows of experts blockIdx.x, blockIdx.x + G, ...
    for (int e = blockIdx.x; e < E; e += G) {
        const int r0 = s_eoff[e] + s_tot[e], r1 = s_eoff[e + 1];
        for (int r = r0 + tid; r < r1; r += kThreads) {
            lp.row_src[r] = -1;
            lp.row_slot[r] = -1;
            if (lp.topk_weights) lp.row_weight[r] = 0.0f;
        }
        for (int r = r0; r < r1 && copy; ++r) {
            uint8_t *o = recv + (int64_t)r * row_bytes;
            for (int v = tid; v < row_bytes / 16; v += kThreads) st_v4(o + v * 16, make_uint4(0, 0, 0, 0));
            if constexpr (FP8)
                for (int b = tid; b < NB; b += kThreads) p.recv_scale[scale_index(p, r, b, NB)] = 0.0f;
        }
    }

    if (blockIdx.x == 0) {
        for (int e = tid; e < E; e += kThreads) {
            lp.cnt[e] = s_tot[e];
            if (lp.u_cnt) lp.u_cnt[e] = s_tot[e];
        }
        for (int e = tid; e <= E; e += kThreads) {
            lp.eoff[e] = s_eoff[e];
            if (lp.u_eoff) lp.u_eoff[e] = s_eoff[e];
        }
        for (int r = tid; r <= R; r += kThreads) {
            lp.roff[r] = s_eoff[r * L];
            if (lp.u_roff) lp.u_roff[r] = s_eoff[r * L];
        }
    }
    if (blockIdx.x == G - 1) {
        // distinct tokens per rank, by the last CTA (s_tot is free now)
        __syncthreads();
        for (int r = tid; r < R; r += kThreads) s_tot[r] = 0;
        __syncthreads();
        for (int t = tid; t < T; t += kThreads) {
            const int64_t *row = idx + (int64_t)t * K;
            if (R <= 64) {
                unsigned long long mask = 0;
                for (int k = 0; k < K; ++k) {
                    const int64_t e = __ldg(row + k);
                    if (e >= 0 && e < E) mask |= 1ull << s_rk[e];
                }
                for (unsigned long long m = mask; m; m &= m - 1) atomicAdd(&s_tot[__ffsll((long long)m) - 1], 1);
            } else {
                for (int k = 0; k < K; ++k) {
                    const int64_t e = __ldg(row + k);
                    if (e < 0 || e >= E) continue;
                    const int r = s_rk[e];
                    bool dup = false;
                    for (int k2 = 0; k2 < k; ++k2) {
                        const int64_t e2 = __ldg(row + k2);
                        if (e2 >= 0 && e2 < E && s_rk[e2] == r) dup = true;
                    }
                    if (!dup) atomicAdd(&s_tot[r], 1);
                }
            }
        }
        __syncthreads();
        for (int r = tid; r < R; r += kThreads) {
            lp.rank_tok[r] = s_tot[r];
            if (lp.u_rank_tok) lp.u_rank_tok[r] = s_tot[r];
        }
    }
}

template <bool FP8, int W>
__global__ void __launch_bounds__(kThreads, 1) layout_dispatch_small_kernel(DispatchParams p, LayoutParams lp) {
    small_layout_dispatch<FP8, W>(p, lp);
}

// The same without the copy (p.x == nullptr): ep_get_layout of a small batch.
__global__ void __launch_bounds__(kThreads, 1) layout_small_kernel(DispatchParams p, LayoutParams lp) {
    small_layout_dispatch<false, 16>(p, lp);
}

}  // namespace

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

// The register kernel: batches too small to fill the GPU (ep_dispatch routes
// larger ones to the chunked kernel of dispatch_lb.cu).
cudaError_t launch_dispatch_bf16(const DispatchParams &p, int num_sms, cudaStream_t s) {
    static OccupancyCache occ16, occ32;
    const bool v32 = (p.H % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    const int units = p.n_token_units + p.n_zero_units;
    if (v32) {
        const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<32, false>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ32), num_sms);
        return launch_pdl(dispatch_bf16_kernel<32, false>, grid, kThreads, 0, s, p);
    }
    const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<16, false>);
    const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ16), num_sms);
    return launch_pdl(dispatch_bf16_kernel<16, false>, grid, kThreads, 0, s, p);
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

// The FP8 register kernel, four resident blocks per SM.
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

// The single-launch layout + dispatch of a small batch (one CTA per token, at
// most num_sms CTAs); with p.x == nullptr the layout alone.
cudaError_t launch_layout_dispatch_small(const DispatchParams &p, const LayoutParams &lp, bool fp8, int num_sms,
                                         cudaStream_t s) {
    const int grid = lp.T < num_sms ? lp.T : num_sms;
    if (p.x == nullptr) {
        layout_small_kernel<<<grid, kThreads, 0, s>>>(p, lp);
        return cudaGetLastError();
    }
    const bool v32 = ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0 &&
                     (fp8 || p.H % 16 == 0);
    if (fp8) {
        if (v32)
            layout_dispatch_small_kernel<true, 32><<<grid, kThreads, 0, s>>>(p, lp);
        else
            layout_dispatch_small_kernel<true, 16><<<grid, kThreads, 0, s>>>(p, lp);
    } else {
        if (v32)
            layout_dispatch_small_kernel<false, 32><<<grid, kThreads, 0, s>>>(p, lp);
        else
            layout_dispatch_small_kernel<false, 16><<<grid, kThreads, 0, s>>>(p, lp);
    }
    return cudaGetLastError();
}

}  // namespace ep
