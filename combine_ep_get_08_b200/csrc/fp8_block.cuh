// fp8_block.cuh -- FP8 E4M3 quantisation of 1x128 blocks of a bf16 row,
// shared by the dispatch kernels that write codes (local and peer-memory).
//
// Per block: a = max(amax, 1e-4), scale = a / 448, code = e4m3_rn_satfinite
// (v * (448 / a)) -- the per-block scaling of "2kiu.com/news/5702702"
// section 2.3 (FP8 transport, one fp32 scale per 128 channels of a token).
#pragma once

#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {

// Two floats -> two E4M3 codes (round to nearest even, saturate to +-448),
// first argument in the low byte.
__device__ __forceinline__ unsigned int e4m3x2(float a, float b) {
    return (unsigned int)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// EPT bf16 elements per thread: load EPT/2 bf16x2 words of a row, store the
// EPT codes (16: 16-byte accesses, 32: 32-byte accesses).
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

// TPB = 128 / EPT consecutive lanes hold one block, NW = EPT / 2 bf16x2 words
// each.  Reduces the block's amax across them with shuffles (every lane of
// the warp takes part), writes the lane's NW / 2 words of codes into q and
// returns the block's scale.
template <int TPB, int NW>
__device__ __forceinline__ float quantize_block(const unsigned int (&w)[NW], unsigned int (&q)[8]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NW; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
#pragma unroll
    for (int o = TPB / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float a = fmaxf(amax, 1e-4f);
    const float inv = 448.0f / a;    // IEEE round-to-nearest divide
#pragma unroll
    for (int i = 0; i < NW / 2; ++i)
        q[i] = e4m3x2(bf16_lo(w[2 * i]) * inv, bf16_hi(w[2 * i]) * inv) |
               (e4m3x2(bf16_lo(w[2 * i + 1]) * inv, bf16_hi(w[2 * i + 1]) * inv) << 16);
    return a / 448.0f;
}

}  // namespace ep
