// combine.cu -- token-major top-k weighted gather-reduce (sm_100a).
//
// out[t, :] = bf16_rn( sum_k w[t,k] * y[pos[t,k], :] ), fp32 accumulation
// with fused multiply-adds in k order from 0.  This is the reverse of
// dispatch: the lesson14_deepep practice task (moe_combine) pulls every
// expert output back to its token and adds weight * output for k = 0..K-1;
// the golden path of bowenzhou.top "deepep/01-overview" section 1.3 maps
// results back through the dispatch handle.
//
// A unit is one column range of one token; every thread issues the K
// independent 16-byte row loads of a column vector before it accumulates,
// so each thread keeps K loads in flight.
#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kThreads = 256;
constexpr int kLoadsInFlight = 8;

__device__ __forceinline__ unsigned int pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const unsigned int *>(&v);
}

__global__ void __launch_bounds__(kThreads) combine_kernel(CombineParams p) {
    __shared__ int32_t s_src[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const int V = p.H / 8;
    const int vps = (V + p.splits - 1) / p.splits;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    uint4 *out = static_cast<uint4 *>(p.out);
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int t = u / p.splits, s = u - t * p.splits;
        if (threadIdx.x < p.K) {
            s_src[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            s_w[threadIdx.x] = __ldg(&p.w[(int64_t)t * p.K + threadIdx.x]);
        }
        __syncthreads();
        const int v0 = s * vps, v1 = min(V, v0 + vps);
        for (int v = v0 + threadIdx.x; v < v1; v += kThreads) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
            for (int k0 = 0; k0 < p.K; k0 += kLoadsInFlight) {
                uint4 yv[kLoadsInFlight];
#pragma unroll
                for (int j = 0; j < kLoadsInFlight; ++j) {
                    const int k = k0 + j;
                    const int src = k < p.K ? s_src[k] : -1;
                    yv[j] = src >= 0 ? ld_stream_v4(y + (int64_t)src * V + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int j = 0; j < kLoadsInFlight; ++j) {
                    const int k = k0 + j;
                    if (k >= p.K || s_src[k] < 0) continue;
                    const float wk = s_w[k];
                    acc[0] = fmaf(wk, bf16_lo(yv[j].x), acc[0]);
                    acc[1] = fmaf(wk, bf16_hi(yv[j].x), acc[1]);
                    acc[2] = fmaf(wk, bf16_lo(yv[j].y), acc[2]);
                    acc[3] = fmaf(wk, bf16_hi(yv[j].y), acc[3]);
                    acc[4] = fmaf(wk, bf16_lo(yv[j].z), acc[4]);
                    acc[5] = fmaf(wk, bf16_hi(yv[j].z), acc[5]);
                    acc[6] = fmaf(wk, bf16_lo(yv[j].w), acc[6]);
                    acc[7] = fmaf(wk, bf16_hi(yv[j].w), acc[7]);
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_v4(out + (int64_t)t * V + v, o);
        }
        __syncthreads();
    }
}

}  // namespace

int combine_threads() { return kThreads; }
const void *combine_kernel_ptr(int) { return reinterpret_cast<const void *>(&combine_kernel); }

cudaError_t launch_combine(const CombineParams &p, int grid, cudaStream_t s) {
    combine_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
