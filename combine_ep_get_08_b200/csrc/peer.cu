// peer.cu -- dispatch and combine straight into / out of other GPUs' buffers
// (sm_100a; expert parallelism across the GPUs of a node over NVLink).
//
// The exchange step of DeepEP's normal mode without a separate all_to_all
// ("blog.hotdry.top ... deepep-expert-parallel-alltoall", first section: the
// normal kernels forward tokens over NVLink inside a node;
// "bowenzhou.top/repos/deepep/01-overview" section 1.3: dispatch, experts,
// combine(x, handle)).  This rank's layout (num_ranks = the number of GPUs)
// makes the rows bound for rank r one contiguous segment
// [rank_offsets[r], rank_offsets[r+1]).  Rank r's receive buffer holds the
// segments of all source ranks one after another; this source's block
// starts at row row0[r] of it.  The dispatch gather stores each row of x
// directly at
//     base[r] + (row0[r] + row - rank_offsets[r]) * row_bytes,
// base[r] being rank r's buffer mapped into this process (CUDA IPC; this
// GPU's own buffer for r == this rank), so the copy to the other GPU is the
// gather's own store stream -- no staging buffer, no second pass.  The FP8
// form quantises each 1x128 block once (the block step shared with the
// local FP8 dispatch) and stores the E4M3 codes and the block's scale into
// the destination's code and scale rows.  The combine reads the expert
// outputs back from the same places and reduces them as ep_combine does.
// Plain loads and stores only: no TMA, no multicast, no wait on another GPU
// (the caller orders the ranks on the host).
#include <cuda_bf16.h>

#include "fp8_block.cuh"
#include "peer.cuh"

namespace ep {

namespace {

constexpr int kPThreads = 256;
constexpr int kPLoadsInFlight = 8;   // row loads a thread issues before it accumulates

__device__ __forceinline__ unsigned int pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const unsigned int *>(&v);
}

struct PeerParams {
    const uint8_t *x;              // [T, H] bf16 (dispatch)
    uint8_t *const *base;          // [R] receive / expert-output buffers
    float *const *sbase;           // [R] scale buffers (FP8 dispatch), else null
    const int32_t *row0;           // [R] first row of this source's block in each
    const int32_t *pos;            // [T, K]
    const int32_t *row_src;        // [cap]
    const int32_t *roff;           // [R+1]
    const float *w;                // [T, K] (combine)
    uint8_t *out;                  // [T, H] bf16 (combine)
    int T, K, R, H;
    int splits;                    // column ranges per token
    int prefetch_x;                // dispatch: pull this CTA's x rows into L2 first (evict_last)
};

// Per-rank addressing, staged in shared memory once per CTA (layout of
// peer_smem_bytes: R row-buffer bases, R scale-buffer bases, row0, roff).
struct PeerTable {
    uint8_t **base;                // [R]
    float **sbase;                 // [R] (FP8 dispatch)
    int32_t *row0;                 // [R]
    int32_t *roff;                 // [R+1]
};

__device__ __forceinline__ PeerTable load_table(const PeerParams &p, unsigned char *smem) {
    PeerTable t;
    t.base = reinterpret_cast<uint8_t **>(smem);
    t.sbase = reinterpret_cast<float **>(smem + sizeof(void *) * p.R);
    t.row0 = reinterpret_cast<int32_t *>(smem + 2 * sizeof(void *) * p.R);
    t.roff = t.row0 + p.R;
    for (int i = threadIdx.x; i < p.R; i += blockDim.x) {
        t.base[i] = p.base[i];
        t.sbase[i] = p.sbase ? p.sbase[i] : nullptr;
        t.row0[i] = __ldg(&p.row0[i]);
    }
    for (int i = threadIdx.x; i <= p.R; i += blockDim.x) t.roff[i] = __ldg(&p.roff[i]);
    __syncthreads();
    return t;
}

// Rank whose segment holds `row`: the largest r with roff[r] <= row (empty
// segments share their start with the next one, so they are skipped).
__device__ __forceinline__ int rank_of_row(const int32_t *roff, int R, int row) {
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (roff[mid] <= row)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Where this rank's received row `row` lives: destination rank and row index there.
struct PeerSlot {
    int r;
    int row;
};

__device__ __forceinline__ PeerSlot peer_slot(const PeerTable &t, int R, int row) {
    const int r = rank_of_row(t.roff, R, row);
    return PeerSlot{r, t.row0[r] + row - t.roff[r]};
}

// Address of this rank's received row `row` in its destination's buffer.
__device__ __forceinline__ uint8_t *peer_row(const PeerTable &t, int R, int row, int row_bytes) {
    const PeerSlot sl = peer_slot(t, R, row);
    return t.base[sl.r] + (int64_t)sl.row * row_bytes;
}

// Units [0, T*splits): one column range of one token to its K rows;
// units after that: the padding rows among 8 consecutive received rows.
__global__ void __launch_bounds__(kPThreads) dispatch_peer_kernel(PeerParams p, int n_zero_units) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ uint8_t *s_dst[kMaxTopk];
    const PeerTable tab = load_table(p, smem);
    const int row_bytes = p.H * 2, nv = row_bytes / 16;
    const int vps = (nv + p.splits - 1) / p.splits;
    const int n_token_units = p.T * p.splits;
    const int rows = tab.roff[p.R];
    if (p.prefetch_x && threadIdx.x == 0) {
        // this CTA's parts of x into L2 first, so that each part's row loads hit there
        const uint64_t pol_x = policy_evict_last();
        for (int u = blockIdx.x; u < n_token_units; u += gridDim.x) {
            const int t = u / p.splits, s = u - t * p.splits;
            const int v0 = s * vps, v1 = min(nv, v0 + vps);
            if (v1 > v0) bulk_prefetch_l2(p.x + (int64_t)t * row_bytes + (int64_t)v0 * 16, (uint32_t)(v1 - v0) * 16, pol_x);
        }
    }
    const uint64_t pol_st = policy_evict_first();   // the received rows are not read again here
    for (int u = blockIdx.x; u < n_token_units + n_zero_units; u += gridDim.x) {
        if (u < n_token_units) {
            const int t = u / p.splits, s = u - t * p.splits;
            const int v0 = s * vps, v1 = min(nv, v0 + vps);
            const uint8_t *xr = p.x + (int64_t)t * row_bytes;
            // the first vector is requested before the destinations are known,
            // so the two memory round trips overlap
            const int vfirst = v0 + threadIdx.x;
            uint4 first = make_uint4(0, 0, 0, 0);
            if (vfirst < v1) first = ld_stream_v4(xr + (int64_t)vfirst * 16);
            if (threadIdx.x < p.K) {
                const int d = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
                s_dst[threadIdx.x] = d >= 0 ? peer_row(tab, p.R, d, row_bytes) : nullptr;
            }
            __syncthreads();
            for (int v = vfirst; v < v1; v += kPThreads) {
                const uint4 val = v == vfirst ? first : ld_stream_v4(xr + (int64_t)v * 16);
                for (int k = 0; k < p.K; ++k)
                    if (s_dst[k]) st_v4_policy(s_dst[k] + (int64_t)v * 16, val, pol_st);
            }
            __syncthreads();
        } else {
            const int r0 = (u - n_token_units) * kZeroRowsPerUnit, r1 = min(rows, r0 + kZeroRowsPerUnit);
            for (int r = r0; r < r1; ++r) {
                if (__ldg(&p.row_src[r]) >= 0) continue;
                uint8_t *o = peer_row(tab, p.R, r, row_bytes);
                for (int v = threadIdx.x; v < nv; v += kPThreads) st_v4(o + (int64_t)v * 16, make_uint4(0, 0, 0, 0));
            }
        }
    }
}

// FP8 dispatch into peer buffers: one token per unit; 8 lanes quantise one
// 1x128 block (16 elements each, 16-byte stores), then store its codes and,
// from the block's first lane, its scale into each of the K destination rows.
// Units after the tokens: padding rows (codes 0, scales 0).
__global__ void __launch_bounds__(kPThreads) dispatch_fp8_peer_kernel(PeerParams p, int n_zero_units) {
    constexpr int EPT = 16, TPB = 128 / EPT, NW = EPT / 2;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ uint8_t *s_dst[kMaxTopk];
    __shared__ float *s_sc[kMaxTopk];
    const PeerTable tab = load_table(p, smem);
    const int NB = p.H / 128, nthr_row = p.H / EPT;
    const int rows = tab.roff[p.R];
    // (an L2 prefetch of the CTA's rows first, as the bf16 kernel does, measured
    // slower here: skew 92.2 -> 98.3 us)
    for (int u = blockIdx.x; u < p.T + n_zero_units; u += gridDim.x) {
        if (u < p.T) {
            const uint8_t *xr = p.x + (int64_t)u * p.H * 2;
            unsigned int w[NW];
            if (threadIdx.x < nthr_row) {
                Fp8Io<EPT>::load(xr + (int64_t)threadIdx.x * EPT * 2, w);
            } else {
#pragma unroll
                for (int i = 0; i < NW; ++i) w[i] = 0;
            }
            if (threadIdx.x < p.K) {
                const int d = __ldg(&p.pos[(int64_t)u * p.K + threadIdx.x]);
                if (d >= 0) {
                    const PeerSlot sl = peer_slot(tab, p.R, d);
                    s_dst[threadIdx.x] = tab.base[sl.r] + (int64_t)sl.row * p.H;
                    s_sc[threadIdx.x] = tab.sbase[sl.r] + (int64_t)sl.row * NB;
                } else {
                    s_dst[threadIdx.x] = nullptr;
                    s_sc[threadIdx.x] = nullptr;
                }
            }
            __syncthreads();
            for (int g0 = 0; g0 < nthr_row; g0 += kPThreads) {      // uniform trip count: every lane shuffles
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
                        if (!s_dst[k]) continue;
                        Fp8Io<EPT>::store(s_dst[k] + (int64_t)g * EPT, q);
                        if (lead) s_sc[k][b] = scale;
                    }
                }
            }
            __syncthreads();
        } else {
            const int r0 = (u - p.T) * kZeroRowsPerUnit, r1 = min(rows, r0 + kZeroRowsPerUnit);
            for (int r = r0; r < r1; ++r) {
                if (__ldg(&p.row_src[r]) >= 0) continue;
                const PeerSlot sl = peer_slot(tab, p.R, r);
                uint8_t *o = tab.base[sl.r] + (int64_t)sl.row * p.H;
                float *sc = tab.sbase[sl.r] + (int64_t)sl.row * NB;
                for (int v = threadIdx.x; v < p.H / 16; v += kPThreads) st_v4(o + (int64_t)v * 16, make_uint4(0, 0, 0, 0));
                for (int b = threadIdx.x; b < NB; b += kPThreads) sc[b] = 0.0f;
            }
        }
    }
}

// out[t] = bf16_rn(sum_k w[t,k] * y[row of (t,k)]), the rows read where the dispatch put them.
__global__ void __launch_bounds__(kPThreads) combine_peer_kernel(PeerParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ const uint8_t *s_src[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const PeerTable tab = load_table(p, smem);
    const int row_bytes = p.H * 2, nv = row_bytes / 16;
    const int vps = (nv + p.splits - 1) / p.splits;
    for (int u = blockIdx.x; u < p.T * p.splits; u += gridDim.x) {
        const int t = u / p.splits, s = u - t * p.splits;
        if (threadIdx.x < p.K) {
            const int d = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            s_src[threadIdx.x] = d >= 0 ? peer_row(tab, p.R, d, row_bytes) : nullptr;
            s_w[threadIdx.x] = __ldg(&p.w[(int64_t)t * p.K + threadIdx.x]);
        }
        __syncthreads();
        const int v0 = s * vps, v1 = min(nv, v0 + vps);
        for (int v = v0 + threadIdx.x; v < v1; v += kPThreads) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
            // fp32 fused multiply-adds in k order from 0; up to kPLoadsInFlight
            // remote loads issued before they are used (NVLink latency)
            for (int k0 = 0; k0 < p.K; k0 += kPLoadsInFlight) {
                uint4 y[kPLoadsInFlight];
#pragma unroll
                for (int j = 0; j < kPLoadsInFlight; ++j)
                    if (k0 + j < p.K && s_src[k0 + j]) y[j] = ld_stream_v4(s_src[k0 + j] + (int64_t)v * 16);
#pragma unroll
                for (int j = 0; j < kPLoadsInFlight; ++j) {
                    if (k0 + j >= p.K || !s_src[k0 + j]) continue;
                    const unsigned int yw[4] = {y[j].x, y[j].y, y[j].z, y[j].w};
                    const float wk = s_w[k0 + j];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[2 * i] = fmaf(wk, bf16_lo(yw[i]), acc[2 * i]);
                        acc[2 * i + 1] = fmaf(wk, bf16_hi(yw[i]), acc[2 * i + 1]);
                    }
                }
            }
            unsigned int o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
            st_v4(p.out + (int64_t)t * row_bytes + (int64_t)v * 16, make_uint4(o[0], o[1], o[2], o[3]));
        }
        __syncthreads();
    }
}

int peer_splits(int T, int num_sms, int nv) {
    int sp = 1;
    while (sp < 8 && T * sp < 2 * num_sms && nv / (sp * 2) >= kPThreads / 2) sp *= 2;
    return sp;
}

}  // namespace

cudaError_t launch_dispatch_peer(const PeerLaunch &l, int num_sms, cudaStream_t s) {
    PeerParams p{};
    p.x = static_cast<const uint8_t *>(l.x);
    p.base = reinterpret_cast<uint8_t *const *>(l.base);
    p.row0 = l.row0;
    p.pos = l.pos;
    p.row_src = l.row_src;
    p.roff = l.roff;
    p.T = l.T;
    p.K = l.K;
    p.R = l.R;
    p.H = l.H;
    p.splits = peer_splits(l.T, num_sms, l.H * 2 / 16);
    p.prefetch_x = l.prefetch_x;
    const int n_zero = l.zero_rows ? (int)((l.cap + kZeroRowsPerUnit - 1) / kZeroRowsPerUnit) : 0;
    const int units = p.T * p.splits + n_zero;
    const int grid = units < 4 * num_sms ? units : 4 * num_sms;
    dispatch_peer_kernel<<<grid, kPThreads, peer_smem_bytes(l.R), s>>>(p, n_zero);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8_peer(const PeerLaunch &l, int num_sms, cudaStream_t s) {
    PeerParams p{};
    p.x = static_cast<const uint8_t *>(l.x);
    p.base = reinterpret_cast<uint8_t *const *>(l.base);
    p.sbase = l.sbase;
    p.row0 = l.row0;
    p.pos = l.pos;
    p.row_src = l.row_src;
    p.roff = l.roff;
    p.T = l.T;
    p.K = l.K;
    p.R = l.R;
    p.H = l.H;
    const int n_zero = l.zero_rows ? (int)((l.cap + kZeroRowsPerUnit - 1) / kZeroRowsPerUnit) : 0;
    const int units = p.T + n_zero;
    const int grid = units < 4 * num_sms ? units : 4 * num_sms;
    dispatch_fp8_peer_kernel<<<grid, kPThreads, peer_smem_bytes(l.R), s>>>(p, n_zero);
    return cudaGetLastError();
}

cudaError_t launch_combine_peer(const PeerLaunch &l, int num_sms, cudaStream_t s) {
    PeerParams p{};
    p.base = reinterpret_cast<uint8_t *const *>(l.base);
    p.row0 = l.row0;
    p.pos = l.pos;
    p.roff = l.roff;
    p.w = l.w;
    p.out = static_cast<uint8_t *>(l.out);
    p.T = l.T;
    p.K = l.K;
    p.R = l.R;
    p.H = l.H;
    p.splits = peer_splits(l.T, num_sms, l.H * 2 / 16);
    const int units = p.T * p.splits;
    const int grid = units < 4 * num_sms ? units : 4 * num_sms;
    combine_peer_kernel<<<grid, kPThreads, peer_smem_bytes(l.R), s>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
