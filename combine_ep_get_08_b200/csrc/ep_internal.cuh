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
constexpr int kLayoutThreads = 512;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kMinTokensPerChunk = 16;
constexpr int kZeroRowsPerUnit = 8;    // padding rows zero-filled per work unit
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;

struct GridBarrier {
    unsigned int count;
    unsigned int gen;
};

// ---------------------------------------------------------------------------
// Kernel parameter blocks
// ---------------------------------------------------------------------------
struct LayoutParams {
    const int64_t *topk_idx;
    const float *topk_weights;   // may be null
    int T, K, E, R, L, A;
    int G;                       // CTAs == chunks
    int tokens_per_chunk;
    // handle arrays
    int32_t *pos, *row_src, *row_slot;
    float *row_weight;
    int32_t *cnt, *rank_tok, *eoff, *roff;
    // caller copies (may be null)
    int32_t *u_cnt, *u_rank_tok, *u_eoff, *u_roff;
    uint8_t *u_in_rank;
    // scratch
    int32_t *chunk_counts;       // [G][E+R]
    int32_t *col_total;          // [E+R]
    GridBarrier *barrier;
    unsigned int *status;
    unsigned long long wait_limit_ns;
    int barrier_extra;
};

struct DispatchParams {
    const void *x;               // [T, H] bf16
    void *recv;                  // [cap, H] bf16 or e4m3
    float *recv_scale;           // [cap, H/128] (FP8 only)
    const int32_t *pos;          // [T, K]
    const int32_t *row_src;      // [cap]
    const int32_t *eoff;         // [E+1]
    int T, K, E, H;
    int splits;                  // column splits per token
    int n_token_units;           // T * splits
    int n_zero_units;            // ceil(cap / kZeroRowsPerUnit) when A > 1, else 0
};

struct CombineParams {
    const void *y;               // [cap, H] bf16
    const float *w;              // [T, K]
    void *out;                   // [T, H] bf16
    const int32_t *pos;          // [T, K]
    int T, K, H;
    int splits;
    int n_units;
};

// launchers (return cudaError_t of the launch)
cudaError_t launch_layout(const LayoutParams &p, size_t smem, cudaStream_t s);
size_t layout_smem_bytes(int E, int R);
const void *layout_kernel_ptr();
cudaError_t launch_dispatch_bf16(const DispatchParams &p, int grid, cudaStream_t s);
cudaError_t launch_dispatch_fp8(const DispatchParams &p, int grid, cudaStream_t s);
cudaError_t launch_combine(const CombineParams &p, int grid, cudaStream_t s);
int dispatch_threads();
int combine_threads();
const void *dispatch_bf16_kernel_ptr();
const void *dispatch_fp8_kernel_ptr();
const void *combine_kernel_ptr(int K);

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

// bf16 pair in a 32-bit word -> two floats (exact)
__device__ __forceinline__ float bf16_lo(unsigned int u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(unsigned int u) { return __uint_as_float(u & 0xffff0000u); }

}  // namespace ep

// The opaque handle.
struct ep_handle {
    ep_config cfg;
    int device;
    int num_sms;
    int64_t cap;
    // layout launch shape
    int G;
    int tokens_per_chunk;
    size_t layout_smem;
    // persistent grids
    int dispatch_grid;
    int dispatch_fp8_grid;
    int combine_grid;
    // one device allocation, carved
    void *block;
    size_t block_bytes;
    int32_t *pos, *row_src, *row_slot;
    float *row_weight;
    int32_t *cnt, *rank_tok, *eoff, *roff;
    int32_t *chunk_counts, *col_total;
    ep::GridBarrier *barrier;
    unsigned int *status;
    bool has_layout;
    unsigned long long wait_limit_ns;
    int barrier_extra;
};
