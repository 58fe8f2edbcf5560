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
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kThreads = 256;

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
    static __device__ __forceinline__ T zero() { return make_uint4(0, 0, 0, 0); }
};
template <>
struct Vec<32> {
    using T = u32x8;
    static __device__ __forceinline__ T load(const void *p) { return ld_stream_v8(p); }
    static __device__ __forceinline__ void store(void *p, const T &v) { st_v8(p, v); }
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

template <int VB>
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
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        if (u < p.n_token_units) {
            const int t = u / p.splits, s = u - t * p.splits;
            if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            __syncthreads();
            const int v0 = s * vps, v1 = min(nv, v0 + vps);
            const uint8_t *xr = x + (int64_t)t * row_bytes;
            for (int v = v0 + threadIdx.x; v < v1; v += kThreads * kUnroll) {
                VT buf[kUnroll];
#pragma unroll
                for (int j = 0; j < kUnroll; ++j)
                    if (v + j * kThreads < v1) buf[j] = V::load(xr + (int64_t)(v + j * kThreads) * VB);
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

// Two floats -> two E4M3 codes (round to nearest even, saturate to +-448),
// first argument in the low byte.
__device__ __forceinline__ unsigned int e4m3x2(float a, float b) {
    return (unsigned int)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// EPT bf16 elements per thread (16: 16-byte accesses, 32: 32-byte accesses);
// TPB = 128 / EPT consecutive lanes share one 1x128 block and reduce its
// amax with shuffles.  Each thread stores EPT code bytes per received row.
template <int EPT>
struct Fp8Io;
template <>
struct Fp8Io<16> {
    static __device__ __forceinline__ void load(const uint8_t *src, unsigned int (&w)[8]) {
        const uint4 a = ld_stream_v4(src), b = ld_stream_v4(src + 16);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
    static __device__ __forceinline__ void store(uint8_t *dst, const unsigned int (&q)[8]) {
        st_v4(dst, make_uint4(q[0], q[1], q[2], q[3]));
    }
};
template <>
struct Fp8Io<32> {
    static __device__ __forceinline__ void load(const uint8_t *src, unsigned int (&w)[16]) {
        const u32x8 a = ld_stream_v8(src), b = ld_stream_v8(src + 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w[i] = a.v[i];
            w[8 + i] = b.v[i];
        }
    }
    static __device__ __forceinline__ void store(uint8_t *dst, const unsigned int (&q)[8]) {
        u32x8 v;
#pragma unroll
        for (int i = 0; i < 8; ++i) v.v[i] = q[i];
        st_v8(dst, v);
    }
};

template <int EPT>
__global__ void __launch_bounds__(kThreads) dispatch_fp8_kernel(DispatchParams p) {
    constexpr int TPB = 128 / EPT;
    constexpr int NW = EPT / 2;              // bf16x2 words loaded per thread
    __shared__ int32_t s_dst[kMaxTopk];
    const int NB = p.H / 128;
    const int nthr_row = p.H / EPT;
    const int total = p.n_token_units + p.n_zero_units;
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    int rows = -1;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        if (u < p.n_token_units) {
            const int t = u;
            if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            __syncthreads();
            const uint8_t *xr = x + (int64_t)t * p.H * 2;
            for (int g0 = 0; g0 < nthr_row; g0 += kThreads) {
                const int g = g0 + threadIdx.x;
                const bool act = g < nthr_row;
                unsigned int w[NW];
                if (act) {
                    Fp8Io<EPT>::load(xr + (int64_t)g * EPT * 2, w);
                } else {
#pragma unroll
                    for (int i = 0; i < NW; ++i) w[i] = 0;
                }
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < NW; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
#pragma unroll
                for (int o = TPB / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const float a = fmaxf(amax, 1e-4f);
                const float inv = 448.0f / a;    // IEEE round-to-nearest divide
                const float scale = a / 448.0f;
                unsigned int q[8];
#pragma unroll
                for (int i = 0; i < NW / 2; ++i)
                    q[i] = e4m3x2(bf16_lo(w[2 * i]) * inv, bf16_hi(w[2 * i]) * inv) |
                           (e4m3x2(bf16_lo(w[2 * i + 1]) * inv, bf16_hi(w[2 * i + 1]) * inv) << 16);
                if (act) {
                    const int b = g / TPB;
                    const bool lead = (g % TPB) == 0;
                    for (int k = 0; k < p.K; ++k) {
                        const int dst = s_dst[k];
                        if (dst < 0) continue;
                        Fp8Io<EPT>::store(recv + (int64_t)dst * p.H + (int64_t)g * EPT, q);
                        if (lead) p.recv_scale[(int64_t)dst * NB + b] = scale;
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
                for (int b = threadIdx.x; b < NB; b += kThreads) p.recv_scale[(int64_t)r * NB + b] = 0.0f;
            }
        }
    }
}

}  // namespace


cudaError_t launch_dispatch_bf16(const DispatchParams &p, int num_sms, cudaStream_t s) {
    static int occ16 = 0, occ32 = 0;
    const int units = p.n_token_units + p.n_zero_units;
    const bool v32 = (p.H % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    if (v32) {
        const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<32>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ32), num_sms);
        dispatch_bf16_kernel<32><<<grid, kThreads, 0, s>>>(p);
    } else {
        const void *k = reinterpret_cast<const void *>(&dispatch_bf16_kernel<16>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ16), num_sms);
        dispatch_bf16_kernel<16><<<grid, kThreads, 0, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8(const DispatchParams &p, int num_sms, cudaStream_t s) {
    static int occ16 = 0, occ32 = 0;
    const int units = p.n_token_units + p.n_zero_units;
    const bool v32 = ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.recv)) & 31) == 0;
    if (v32) {
        const void *k = reinterpret_cast<const void *>(&dispatch_fp8_kernel<32>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ32), num_sms);
        dispatch_fp8_kernel<32><<<grid, kThreads, 0, s>>>(p);
    } else {
        const void *k = reinterpret_cast<const void *>(&dispatch_fp8_kernel<16>);
        const int grid = persistent_grid(units, blocks_per_sm(k, kThreads, 0, &occ16), num_sms);
        dispatch_fp8_kernel<16><<<grid, kThreads, 0, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace ep
