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
// consecutive received rows (only when expert_alignment > 1).
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // 16-byte vectors in flight per thread (bf16 path)

__global__ void __launch_bounds__(kThreads) dispatch_bf16_kernel(DispatchParams p) {
    __shared__ int32_t s_dst[kMaxTopk];
    const int V = p.H / 8;                      // 16-byte vectors per row
    const int vps = (V + p.splits - 1) / p.splits;
    const int total = p.n_token_units + p.n_zero_units;
    const uint4 *x = static_cast<const uint4 *>(p.x);
    uint4 *recv = static_cast<uint4 *>(p.recv);
    int rows = -1;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        if (u < p.n_token_units) {
            const int t = u / p.splits, s = u - t * p.splits;
            if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            __syncthreads();
            const int v0 = s * vps, v1 = min(V, v0 + vps);
            const uint4 *xr = x + (int64_t)t * V;
            for (int v = v0 + threadIdx.x; v < v1; v += kThreads * kUnroll) {
                uint4 buf[kUnroll];
#pragma unroll
                for (int j = 0; j < kUnroll; ++j)
                    if (v + j * kThreads < v1) buf[j] = ld_stream_v4(xr + v + j * kThreads);
                for (int k = 0; k < p.K; ++k) {
                    const int dst = s_dst[k];
                    if (dst < 0) continue;
                    uint4 *o = recv + (int64_t)dst * V;
#pragma unroll
                    for (int j = 0; j < kUnroll; ++j)
                        if (v + j * kThreads < v1) st_v4(o + v + j * kThreads, buf[j]);
                }
            }
            __syncthreads();
        } else {
            if (rows < 0) rows = __ldg(&p.eoff[p.E]);
            const int r0 = (u - p.n_token_units) * kZeroRowsPerUnit;
            const int r1 = min(rows, r0 + kZeroRowsPerUnit);
            for (int r = r0; r < r1; ++r) {
                if (__ldg(&p.row_src[r]) >= 0) continue;
                uint4 *o = recv + (int64_t)r * V;
                for (int v = threadIdx.x; v < V; v += kThreads) st_v4(o + v, make_uint4(0, 0, 0, 0));
            }
        }
    }
}

// Two floats -> two E4M3 codes (round to nearest even, saturate to +-448),
// first argument in the low byte.
__device__ __forceinline__ unsigned int e4m3x2(float a, float b) {
    return (unsigned int)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(kThreads) dispatch_fp8_kernel(DispatchParams p) {
    __shared__ int32_t s_dst[kMaxTopk];
    const int NB = p.H / 128;                   // 1x128 blocks per row
    const int bps = (NB + p.splits - 1) / p.splits;
    const int total = p.n_token_units + p.n_zero_units;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, l16 = lane & 15;
    constexpr int NW = kThreads / 32;
    const uint4 *x = static_cast<const uint4 *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    int rows = -1;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        if (u < p.n_token_units) {
            const int t = u / p.splits, s = u - t * p.splits;
            if (threadIdx.x < p.K) s_dst[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            __syncthreads();
            const int b0 = s * bps, b1 = min(NB, b0 + bps);
            const uint4 *xr = x + (int64_t)t * (p.H / 8);
            // each half-warp owns one 128-column block per iteration
            for (int bp = b0 + 2 * warp; bp < b1; bp += 2 * NW) {
                const int b = bp + half;
                const bool act = b < b1;
                const uint4 xv = act ? ld_stream_v4(xr + b * 16 + l16) : make_uint4(0, 0, 0, 0);
                const float f0 = bf16_lo(xv.x), f1 = bf16_hi(xv.x), f2 = bf16_lo(xv.y), f3 = bf16_hi(xv.y);
                const float f4 = bf16_lo(xv.z), f5 = bf16_hi(xv.z), f6 = bf16_lo(xv.w), f7 = bf16_hi(xv.w);
                float amax = fmaxf(fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3))),
                                   fmaxf(fmaxf(fabsf(f4), fabsf(f5)), fmaxf(fabsf(f6), fabsf(f7))));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const float a = fmaxf(amax, 1e-4f);
                const float inv = 448.0f / a;    // IEEE round-to-nearest divide
                const float scale = a / 448.0f;
                uint2 q;
                q.x = e4m3x2(f0 * inv, f1 * inv) | (e4m3x2(f2 * inv, f3 * inv) << 16);
                q.y = e4m3x2(f4 * inv, f5 * inv) | (e4m3x2(f6 * inv, f7 * inv) << 16);
                if (act) {
                    for (int k = 0; k < p.K; ++k) {
                        const int dst = s_dst[k];
                        if (dst < 0) continue;
                        st_v2(recv + (int64_t)dst * p.H + b * 128 + l16 * 8, q);
                        if (l16 == 0) p.recv_scale[(int64_t)dst * NB + b] = scale;
                    }
                }
            }
            __syncthreads();
        } else {
            if (rows < 0) rows = __ldg(&p.eoff[p.E]);
            const int r0 = (u - p.n_token_units) * kZeroRowsPerUnit;
            const int r1 = min(rows, r0 + kZeroRowsPerUnit);
            const int V = p.H / 16;
            for (int r = r0; r < r1; ++r) {
                if (__ldg(&p.row_src[r]) >= 0) continue;
                uint4 *o = reinterpret_cast<uint4 *>(recv + (int64_t)r * p.H);
                for (int v = threadIdx.x; v < V; v += kThreads) st_v4(o + v, make_uint4(0, 0, 0, 0));
                for (int b = threadIdx.x; b < NB; b += kThreads) p.recv_scale[(int64_t)r * NB + b] = 0.0f;
            }
        }
    }
}

}  // namespace

int dispatch_threads() { return kThreads; }
const void *dispatch_bf16_kernel_ptr() { return reinterpret_cast<const void *>(&dispatch_bf16_kernel); }
const void *dispatch_fp8_kernel_ptr() { return reinterpret_cast<const void *>(&dispatch_fp8_kernel); }

cudaError_t launch_dispatch_bf16(const DispatchParams &p, int grid, cudaStream_t s) {
    dispatch_bf16_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8(const DispatchParams &p, int grid, cudaStream_t s) {
    dispatch_fp8_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
