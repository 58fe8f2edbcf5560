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

// NW = bf16x2 words per vector (4: 16-byte loads; a 32-byte variant needs
// ~100 registers, halves occupancy and measured slower).
template <int NW>
struct CVec;
template <>
struct CVec<4> {
    static __device__ __forceinline__ void load(const void *p, unsigned int (&w)[4]) {
        const uint4 v = ld_stream_v4(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    }
    static __device__ __forceinline__ void store(void *p, const unsigned int (&w)[4]) {
        st_v4(p, make_uint4(w[0], w[1], w[2], w[3]));
    }
};

template <int NW>
// Four resident blocks per SM (62 registers, no spill); three measured 8% slower.
__global__ void __launch_bounds__(kThreads, 4) combine_kernel(CombineParams p) {
    constexpr int VB = NW * 4;               // bytes per vector
    __shared__ int32_t s_src[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const int row_bytes = p.H * 2;
    const int V = row_bytes / VB;
    const int vps = (V + p.splits - 1) / p.splits;
    const uint8_t *y = static_cast<const uint8_t *>(p.y);
    uint8_t *out = static_cast<uint8_t *>(p.out);
    pdl_wait();   // the kernel before (the expert computation) is complete and visible
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int t = u / p.splits, s = u - t * p.splits;
        if (threadIdx.x < p.K) {
            s_src[threadIdx.x] = __ldg(&p.pos[(int64_t)t * p.K + threadIdx.x]);
            s_w[threadIdx.x] = __ldg(&p.w[(int64_t)t * p.K + threadIdx.x]);
        }
        __syncthreads();
        const int v0 = s * vps, v1 = min(V, v0 + vps);
        for (int v = v0 + threadIdx.x; v < v1; v += kThreads) {
            float acc[2 * NW];
#pragma unroll
            for (int i = 0; i < 2 * NW; ++i) acc[i] = 0.0f;
            for (int k0 = 0; k0 < p.K; k0 += kLoadsInFlight) {
                unsigned int yv[kLoadsInFlight][NW];
#pragma unroll
                for (int j = 0; j < kLoadsInFlight; ++j) {
                    const int k = k0 + j;
                    const int src = k < p.K ? s_src[k] : -1;
                    if (src >= 0) {
                        CVec<NW>::load(y + (int64_t)src * row_bytes + (int64_t)v * VB, yv[j]);
                    } else {
#pragma unroll
                        for (int i = 0; i < NW; ++i) yv[j][i] = 0;
                    }
                }
#pragma unroll
                for (int j = 0; j < kLoadsInFlight; ++j) {
                    const int k = k0 + j;
                    if (k >= p.K || s_src[k] < 0) continue;
                    const float wk = s_w[k];
#pragma unroll
                    for (int i = 0; i < NW; ++i) {
                        acc[2 * i] = fmaf(wk, bf16_lo(yv[j][i]), acc[2 * i]);
                        acc[2 * i + 1] = fmaf(wk, bf16_hi(yv[j][i]), acc[2 * i + 1]);
                    }
                }
            }
            unsigned int o[NW];
#pragma unroll
            for (int i = 0; i < NW; ++i) o[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
            CVec<NW>::store(out + (int64_t)t * row_bytes + (int64_t)v * VB, o);
        }
        __syncthreads();
    }
}

}  // namespace

// A staged variant (bulk loads of the K row chunks into a shared-memory
// ring, one consumer group per SM) measured slower (123 vs 80.7 us at the
// DeepSeek-V3 shape): the fp32 accumulation needs the register kernel's
// four resident blocks per SM.
cudaError_t launch_combine(const CombineParams &p_in, int num_sms, cudaStream_t s) {
    static OccupancyCache occ;
    CombineParams p = p_in;
    // a small batch splits each row over several CTAs (at least half a
    // block of vectors each) so that it still spreads over the SMs
    const int nv = p.H * 2 / 16;
    int sp = 1;
    while (sp < 8 && p.T * sp < 2 * num_sms && nv / (sp * 2) >= kThreads / 2) sp *= 2;
    p.splits = sp;
    p.n_units = p.T * sp;
    const void *k = reinterpret_cast<const void *>(&combine_kernel<4>);
    const int grid = persistent_grid(p.n_units, blocks_per_sm(k, kThreads, 0, &occ), num_sms);
    // programmatic stream serialization: the launch may overlap the end of
    // the previous kernel; the kernel waits before its first global read
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel<4>, p);
}

}  // namespace ep
