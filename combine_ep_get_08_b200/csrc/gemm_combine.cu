// gemm_combine.cu -- expert GEMM with the combine fused into its epilogue
// (sm_100a, tcgen05 tensor cores).
//
//   out[t, :] = bf16_rn( sum_k w[t,k] * act[pos[t,k], :] @ W_e^T ),  e = expert of pair (t, k)
//
// The expert step between dispatch and combine ("lesson14_deepep" practice
// task: each expert transforms the rows it received, combine adds
// weight * expert output back into the token's row), for the linear map of
// an expert's last projection.  The rows arrive in the handle's received-row
// layout, whose expert segments are padded to expert_alignment -- with an
// alignment that is a multiple of 128 (EPBuffer.dispatch's
// expert_alignment, bowenzhou.top "deepep/01-overview" section 1.1) every
// 128-row tile belongs to one expert, so the GEMM needs no per-row expert
// lookup.
//
// Persistent grid, one CTA per SM, 192 threads:
//   warp 0     TMA producer: 128x64 tiles of act and 256x64 tiles of W_e
//              (128-byte swizzle) into a 4-stage shared-memory ring;
//   warp 1     allocates 512 TMEM columns (two fp32 128x256 accumulators)
//              and issues tcgen05.mma (M=128, N=256, K=16, bf16 in, fp32
//              accumulate) from one thread; tcgen05.commit frees ring
//              stages and hands finished accumulators to the epilogue;
//   warps 2-5  epilogue, one warp per 32-lane quarter of TMEM (warp w reads
//              lanes 32*(w%4)...): tcgen05.ld a row's columns, scale them by
//              the pair's top-k weight, transpose each 32x32 chunk through
//              shared memory and add it into an fp32 [T, N] accumulator with
//              16-byte vector atomics that cover 128 contiguous bytes per 8
//              lanes -- the combine, fused.  Padding rows add nothing.
// A second kernel rounds the fp32 accumulator to bf16.  Every wait on an
// mbarrier is bounded; a timeout sets EP_DEV_WAIT_TIMEOUT, lets the copies
// and MMAs in flight finish (bounded again), frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kGM = 128;                              // rows per tile
constexpr int kGN = 256;                              // output columns per tile
constexpr int kGK = 64;                               // inner elements per stage: one 128-byte row
constexpr int kGStages = 4;
constexpr uint32_t kGABytes = kGM * kGK * 2;          // 16 KB
constexpr uint32_t kGBBytes = kGN * kGK * 2;          // 32 KB
constexpr int kGEpiWarps = 4;                        // one per TMEM lane quarter (8 measured slower: the
                                                      // atomic adds are bound by L2, not by issue)
constexpr int kGThreads = 64 + 32 * kGEpiWarps;
constexpr int kGAcc = 2;                              // TMEM accumulators
constexpr uint32_t kGTmemCols = kGAcc * kGN;          // 512: all of an SM's TMEM
constexpr uint32_t kGStageT = 32 * 32 * 4;           // one epilogue warp's 32x32 fp32 transpose tile
constexpr size_t kGSmem = 1024 + kGStages * (size_t)(kGABytes + kGBBytes) + kGEpiWarps * kGStageT + 256;

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), bf16 A and B (bits 7-9, 10-12 = 1), both K-major (bits 15, 16 =
// 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kGN >> 3) << 17) |
                             ((uint32_t)(kGM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major tile with 128-byte swizzle:
// rows of 128 bytes, 8-row atoms of 1024 bytes (stride byte offset), start
// address >> 4 in bits 0-13, leading byte offset 1 (unused for this
// layout), version 1 at bit 46, layout type 2 (128-byte swizzle) at 61-63.
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// 2-D tiled TMA load into shared memory (no multicast), completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(a), "l"(b), "r"(kGIdesc), "r"(accumulate));
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :
                 : "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" : : : "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" : : : "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" : : : "memory");
}

// Tiles are numbered expert by expert; inside an expert by column block and
// then by row block, so the CTAs running side by side share one 256-column
// slice of W_e (read from DRAM once, then from L2) and the expert's row
// blocks.  Expert e's tiles start at (eoff[e] / kGM) * n_blocks.
struct GemmTile {
    int m;   // row block (global)
    int n;   // column block
    int e;   // expert
};

__device__ __forceinline__ GemmTile tile_coords(const int32_t *eoff, int E, int n_blocks, int t) {
    int lo = 0, hi = E - 1;   // largest e whose first tile is <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&eoff[mid]) / kGM * n_blocks <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    // an empty expert shares its first tile with the next one, so lo is never empty
    const int m0 = __ldg(&eoff[lo]) / kGM;
    const int mb = __ldg(&eoff[lo + 1]) / kGM - m0;
    const int local = t - m0 * n_blocks;
    GemmTile g;
    g.e = lo;
    g.n = local / mb;
    g.m = m0 + (local - g.n * mb);
    return g;
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_combine_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        GemmCombineParams p) {
    extern __shared__ uint8_t g_smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(g_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + kGStages * kGABytes;
    float *sT = reinterpret_cast<float *>(sB + kGStages * kGBBytes);   // [epilogue warps][32 rows][32 cols], swizzled
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sT) + kGEpiWarps * kGStageT);
    uint64_t *empty = full + kGStages;
    uint64_t *acc_full = empty + kGStages;
    uint64_t *acc_empty = acc_full + kGAcc;
    uint64_t *drain = acc_empty + kGAcc;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = __ldg(&p.eoff[p.E]);
    const int n_blocks = p.N / kGN;
    const int tiles = (rows / kGM) * n_blocks;
    const int k_blocks = p.I / kGK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < kGAcc; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kGEpiWarps);   // lane 0 of each epilogue warp
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :
                     : "r"(smem_u32(s_tmem)), "r"(kGTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" : : : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ---- TMA producer ----
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x) {
                const GemmTile g = tile_coords(p.eoff, p.E, n_blocks, tile);
                const int m = g.m, n = g.n, e = g.e;
                for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                    const int s = it % kGStages, use = it / kGStages;
                    if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1, p.wait_limit_ns)) {
                        atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *s_abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], kGABytes + kGBBytes);
                    tma_load_2d(sA + s * kGABytes, &map_a, kb * kGK, m * kGM, &full[s]);
                    tma_load_2d(sB + s * kGBBytes, &map_b, kb * kGK, e * p.N + n * kGN, &full[s]);
                }
            }
            // on abort, let the loads already issued land before shared memory goes away
            if (*s_abort)
                for (int j = max(0, it - kGStages); j < it; ++j)
                    mbar_wait_bounded(&full[j % kGStages], (j / kGStages) & 1, p.wait_limit_ns);
        }
    } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
            int it = 0, local = 0;
            for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x, ++local) {
                const int acc = local % kGAcc, ause = local / kGAcc;
                if (ause > 0 && !mbar_wait_bounded(&acc_empty[acc], (ause - 1) & 1, p.wait_limit_ns)) {
                    atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * kGN);
                bool ok = true;
                for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                    const int s = it % kGStages;
                    if (!mbar_wait_bounded(&full[s], (it / kGStages) & 1, p.wait_limit_ns)) {
                        atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a = umma_desc_k_sw128(smem_u32(sA + s * kGABytes));
                    const uint64_t b = umma_desc_k_sw128(smem_u32(sB + s * kGBBytes));
#pragma unroll
                    for (int kk = 0; kk < kGK / 16; ++kk)   // 16 bf16 = 32 bytes = 2 descriptor units
                        umma_bf16(d, a + 2 * kk, b + 2 * kk, (kb | kk) != 0);
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
            }
            // every MMA issued has completed before TMEM is freed
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, p.wait_limit_ns);
        }
    } else {
        // ---- epilogue: scale by the pair's weight, add into the token's row ----
        // A thread holds one row (its TMEM lane) of each 32-column chunk; the
        // chunk is transposed through a swizzled shared-memory tile so that
        // eight lanes cover 128 contiguous bytes of one token row and each
        // warp-wide vector add touches 4 rows instead of 32.
        const int q = warp & 3;                    // TMEM lanes 32q .. 32q+31
        constexpr int kChunks = (kGN / 32) / (kGEpiWarps / 4);                  // 32-column chunks per warp
        const int c_lo = (warp - 2) / 4 * kChunks, c_hi = c_lo + kChunks;
        float4 *tile4 = reinterpret_cast<float4 *>(sT + (warp - 2) * (kGStageT / 4));
        int local = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
            const int acc = local % kGAcc, ause = local / kGAcc;
            if (*s_abort || !mbar_wait_bounded(&acc_full[acc], ause & 1, p.wait_limit_ns)) {
                if (!*s_abort) {
                    atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                    *s_abort = 1;
                }
                break;
            }
            tc_fence_after();
            const GemmTile g = tile_coords(p.eoff, p.E, n_blocks, tile);
            const int r = g.m * kGM + q * 32 + lane;
            const int src = __ldg(&p.row_src[r]);
            float wt = 0.0f;
            if (src >= 0) wt = __ldg(&p.topk_w[(int64_t)src * p.K + __ldg(&p.row_slot[r])]);
            const int sub = lane >> 3, k4 = lane & 7;  // reader: row i0 + sub, float4 k4 of the chunk
            for (int c = c_lo; c < c_hi; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kGN + c * 32), v);
#pragma unroll
                for (int k = 0; k < 8; ++k)                 // float4 k of row `lane` at slot k ^ (lane & 7)
                    tile4[lane * 8 + (k ^ (lane & 7))] =
                        make_float4(wt * __uint_as_float(v[4 * k]), wt * __uint_as_float(v[4 * k + 1]),
                                    wt * __uint_as_float(v[4 * k + 2]), wt * __uint_as_float(v[4 * k + 3]));
                __syncwarp();
                float *ocol = p.out_acc + (int64_t)g.n * kGN + c * 32 + k4 * 4;
#pragma unroll
                for (int i0 = 0; i0 < 32; i0 += 4) {
                    const int i = i0 + sub;
                    const int t = __shfl_sync(0xffffffffu, src, i);
                    const float4 val = tile4[i * 8 + (k4 ^ (i & 7))];
                    if (t >= 0) atomicAdd(reinterpret_cast<float4 *>(ocol + (int64_t)t * p.N), val);
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" : : "r"(tmem), "r"(kGTmemCols) : "memory");
}

// ---------------------------------------------------------------------------
// FP8 form: E4M3 rows with one fp32 scale per row and 128 inner elements (what
// the FP8 dispatch writes) times E4M3 expert matrices with one fp32 scale per
// 128 x 128 block ("m.nlpx.cn/news/135159" section 4.1, per-block scaling;
// the grouped FP8 expert GEMM of "lesson14_deepep" section 3):
//   out[t, :] = bf16_rn( sum_k w[t,k] * sum_b sa[r, b] * sw[e, :/128, b] * (q[r, b] . Wq_e[:, b]) ).
// The scales change every 128 inner elements, so they cannot ride inside one
// tensor-core accumulation: each 128-deep k-block is its own tcgen05.mma
// (kind::f8f6f4, M=128, N=256, K=32, four per k-block) into one of two TMEM
// partial buffers, and the epilogue warps fold each partial into fp32
// registers with its two scales (sa of the row, sw of the 128-column half)
// while the tensor cores fill the other buffer.  Twelve warps: warpgroup 0
// holds the TMA producer (warp 0) and the MMA issuer (warp 1); warpgroups 1-2
// are eight epilogue warps, warp w reading TMEM lanes 32*(w%4).. and one
// 128-column half of the tile, so a thread keeps 128 running sums (setmaxnreg
// moves registers from warpgroup 0 to them).  After the tile's last k-block
// the sums are scaled by the pair's top-k weight and added into the token's
// fp32 row as in the bf16 kernel.  Same persistent tile order, producer and
// bounded waits.
// ---------------------------------------------------------------------------
#ifndef EP_F8_TILE_N
#define EP_F8_TILE_N 256     // output columns per tile of the FP8 kernel (TMEM holds 512 / N partial buffers)
#endif
constexpr int kFN = EP_F8_TILE_N;
constexpr int kFBufs = 512 / kFN;                     // TMEM partial buffers
constexpr int kFK = 128;                              // inner elements per stage: one 128-byte row = one scale block
constexpr int kFStages = 4;
constexpr uint32_t kFABytes = kGM * kFK;              // 16 KB
constexpr uint32_t kFBBytes = kFN * kFK;
constexpr int kFEpiWarps = 8;                         // 4 lane quarters x 2 column halves
constexpr int kFEpiWarp0 = 4;                         // epilogue warps are the 2nd and 3rd warpgroups
constexpr int kFThreads = 32 * (kFEpiWarp0 + kFEpiWarps);
// Register split (setmaxnreg, per warpgroup): the launch gives 384 threads x 168;
// the producer warpgroup drops to 40 and the two epilogue warpgroups rise to 232
// (128 x 40 + 256 x 232 = 384 x 168), room for 128 running sums and 64 loaded columns.
constexpr int kFRegsLaunch = 168, kFRegsLow = 40, kFRegsHigh = 232;
static_assert(128 * kFRegsLow + 256 * kFRegsHigh <= kFThreads * kFRegsLaunch, "register split exceeds the launch");
constexpr int kFLdBatch = 4;                          // 16-column TMEM loads in flight per wait
constexpr int kFHalf = kFN / 2;                       // columns per epilogue thread
constexpr uint32_t kFTmemCols = kFBufs * kFN;         // all 512 columns
constexpr size_t kFSmem = 1024 + kFStages * (size_t)(kFABytes + kFBBytes) + kFEpiWarps * kGStageT + 256;

// Instruction descriptor of tcgen05.mma kind::f8f6f4: fp32 accumulator (bits
// 4-5 = 1), E4M3 A and B (format code 0 at bits 7-9 and 10-12), both K-major,
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kFIdesc = (1u << 4) | ((uint32_t)(kFN >> 3) << 17) | ((uint32_t)(kGM >> 4) << 24);

__device__ __forceinline__ void umma_e4m3(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "l"(a), "l"(b), "r"(kFIdesc), "r"(accumulate));
}

// 16 columns of this lane, no wait: the caller waits with tmem_wait_ld and
// then passes the registers through tmem_fence_regs before using them.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t *v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" : : : "memory"); }
// Orders every use of the 16 registers after the preceding (volatile) wait.
__device__ __forceinline__ void tmem_fence_regs(uint32_t *v) {
    asm volatile(""
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]));
}

__global__ void __launch_bounds__(kFThreads, 1)
    gemm_combine_fp8_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                            GemmCombineParams p) {
    extern __shared__ uint8_t g_smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(g_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + kFStages * kFABytes;
    float *sT = reinterpret_cast<float *>(sB + kFStages * kFBBytes);   // [epilogue warps][32 rows][32 cols], swizzled
    uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sT) + kFEpiWarps * kGStageT);
    uint64_t *empty = full + kFStages;
    uint64_t *part_full = empty + kFStages;       // [kFBufs] a k-block's partial product is in TMEM buffer j
    uint64_t *part_empty = part_full + kFBufs;    // [kFBufs] every epilogue warp has read buffer j
    uint64_t *drain = part_empty + kFBufs;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = __ldg(&p.eoff[p.E]);
    const int n_blocks = p.N / kFN;
    const int tiles = (rows / kGM) * n_blocks;
    const int k_blocks = p.I / kFK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < kFBufs; ++j) {
            mbar_init(&part_full[j], 1);
            mbar_init(&part_empty[j], kFEpiWarps);   // lane 0 of each epilogue warp
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_async_smem();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :
                     : "r"(smem_u32(s_tmem)), "r"(kFTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" : : : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    if (warp < kFEpiWarp0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" : : "n"(kFRegsLow));
        if (warp == 0) {
            // ---- TMA producer ----
            if (lane == 0) {
                int it = 0;
                for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x) {
                    const GemmTile g = tile_coords(p.eoff, p.E, n_blocks, tile);
                    for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                        const int s = it % kFStages, use = it / kFStages;
                        if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1, p.wait_limit_ns)) {
                            atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                            *s_abort = 1;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[s], kFABytes + kFBBytes);
                        tma_load_2d(sA + s * kFABytes, &map_a, kb * kFK, g.m * kGM, &full[s]);
                        tma_load_2d(sB + s * kFBBytes, &map_b, kb * kFK, g.e * p.N + g.n * kFN, &full[s]);
                    }
                }
                if (*s_abort)
                    for (int j = max(0, it - kFStages); j < it; ++j)
                        mbar_wait_bounded(&full[j % kFStages], (j / kFStages) & 1, p.wait_limit_ns);
            }
        } else if (warp == 1) {
            // ---- MMA issuer: one partial product per k-block, alternating TMEM buffers ----
            if (lane == 0) {
                int it = 0;
                for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x) {
                    bool ok = true;
                    for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                        const int j = it % kFBufs, juse = it / kFBufs, s = it % kFStages;
                        if (juse > 0 && !mbar_wait_bounded(&part_empty[j], (juse - 1) & 1, p.wait_limit_ns)) {
                            ok = false;
                        } else if (!mbar_wait_bounded(&full[s], (it / kFStages) & 1, p.wait_limit_ns)) {
                            ok = false;
                        }
                        if (!ok) {
                            atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                            *s_abort = 1;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem + (uint32_t)(j * kFN);
                        const uint64_t a = umma_desc_k_sw128(smem_u32(sA + s * kFABytes));
                        const uint64_t b = umma_desc_k_sw128(smem_u32(sB + s * kFBBytes));
    #pragma unroll
                        for (int kk = 0; kk < kFK / 32; ++kk)   // 32 E4M3 = 32 bytes = 2 descriptor units
                            umma_e4m3(d, a + 2 * kk, b + 2 * kk, kk != 0);
                        umma_commit(&empty[s]);
                        umma_commit(&part_full[j]);
                    }
                    if (!ok) break;
                }
                umma_commit(drain);
                mbar_wait_bounded(drain, 0, p.wait_limit_ns);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" : : "n"(kFRegsHigh));
        // ---- epilogue: fold the scaled partials, then combine ----
        const int ew = warp - kFEpiWarp0;
        const int q = warp & 3;                    // TMEM lanes 32q .. 32q+31
        const int h = ew >> 2;                     // column half of the tile
        const int IB = p.I / kFK, NB = p.N / 128;
        float4 *tile4 = reinterpret_cast<float4 *>(sT + ew * (kGStageT / 4));
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kFHalf);
        int it = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const GemmTile g = tile_coords(p.eoff, p.E, n_blocks, tile);
            const int r = g.m * kGM + q * 32 + lane;
            const int src = __ldg(&p.row_src[r]);
            float wt = 0.0f;
            if (src >= 0) wt = __ldg(&p.topk_w[(int64_t)src * p.K + __ldg(&p.row_slot[r])]);
            const float *sa_row = p.scale_ld > 0 ? p.act_scale + r : p.act_scale + (int64_t)r * IB;
            const int64_t sa_step = p.scale_ld > 0 ? p.scale_ld : 1;
            const float *sw_blk = p.w_scale + ((int64_t)g.e * NB + (g.n * kFN + h * kFHalf) / 128) * IB;
            float acc[kFHalf];
#pragma unroll
            for (int c = 0; c < kFHalf; ++c) acc[c] = 0.0f;
            float sa_next = __ldg(sa_row), sw_next = __ldg(sw_blk);
            bool ok = true;
            for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                const float sc = sa_next * sw_next;
                if (kb + 1 < k_blocks) {
                    sa_next = __ldg(sa_row + (kb + 1) * sa_step);
                    sw_next = __ldg(sw_blk + kb + 1);
                }
                const int j = it % kFBufs;
                if (*s_abort || !mbar_wait_bounded(&part_full[j], (it / kFBufs) & 1, p.wait_limit_ns)) {
                    if (!*s_abort) {
                        atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                        *s_abort = 1;
                    }
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < kFHalf / 16; c0 += kFLdBatch) {
                    uint32_t v[kFLdBatch][16];
#pragma unroll
                    for (int c = 0; c < kFLdBatch; ++c)
                        tmem_ld16_async(lane_base + (uint32_t)(j * kFN + (c0 + c) * 16), v[c]);
                    tmem_wait_ld();
                    if (c0 + kFLdBatch >= kFHalf / 16) {
                        // the buffer's last columns are in registers: hand it back before folding
                        // them (one run: 1212 -> 1235 TFLOP/s)
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&part_empty[j]);
                    }
#pragma unroll
                    for (int c = 0; c < kFLdBatch; ++c) {
                        tmem_fence_regs(v[c]);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            acc[(c0 + c) * 16 + i] = fmaf(sc, __uint_as_float(v[c][i]), acc[(c0 + c) * 16 + i]);
                    }
                }
            }
            if (!ok) break;
            // combine: a thread holds one row of 128 columns; each 32-column chunk is
            // transposed through shared memory so eight lanes cover 128 contiguous bytes
            const int sub = lane >> 3, k4 = lane & 7;
#pragma unroll
            for (int c = 0; c < kFHalf / 32; ++c) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tile4[lane * 8 + (k ^ (lane & 7))] =
                        make_float4(wt * acc[c * 32 + 4 * k], wt * acc[c * 32 + 4 * k + 1],
                                    wt * acc[c * 32 + 4 * k + 2], wt * acc[c * 32 + 4 * k + 3]);
                __syncwarp();
                float *ocol = p.out_acc + (int64_t)g.n * kFN + h * kFHalf + c * 32 + k4 * 4;
#pragma unroll
                for (int i0 = 0; i0 < 32; i0 += 4) {
                    const int i = i0 + sub;
                    const int t = __shfl_sync(0xffffffffu, src, i);
                    const float4 val = tile4[i * 8 + (k4 ^ (i & 7))];
                    if (t >= 0) atomicAdd(reinterpret_cast<float4 *>(ocol + (int64_t)t * p.N), val);
                }
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" : : "r"(tmem), "r"(kFTmemCols) : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// out = bf16_rn(acc), 8 elements per thread per step.
__global__ void acc_to_bf16_kernel(const float *acc, void *out, int64_t n8) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = reinterpret_cast<const float4 *>(acc)[2 * i];
        const float4 b = reinterpret_cast<const float4 *>(acc)[2 * i + 1];
        reinterpret_cast<uint4 *>(out)[i] =
            make_uint4(bf16x2_rn(a.x, a.y), bf16x2_rn(a.z, a.w), bf16x2_rn(b.x, b.y), bf16x2_rn(b.z, b.w));
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// A [rows_total, inner] row-major matrix (bf16, or one byte per element when fp8) read in
// (box_rows x 128 bytes) tiles with 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *ptr, int64_t rows_total, int inner, int box_rows, bool fp8) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int esize = fp8 ? 1 : 2;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows_total};
    const cuuint64_t strides[1] = {(cuuint64_t)inner * esize};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / esize), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr),
              dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_combine(const GemmCombineArgs &g, int num_sms, cudaStream_t s) {
    // the kernel attributes belong to each device's context: set them once per device
    static int ready[kMaxDevices];
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE)) {
        cudaError_t e = cudaFuncSetAttribute(gemm_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_combine_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kFSmem);
        if (e != cudaSuccess) return e;
        __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
    }
    CUtensorMap map_a, map_b;
    if (!make_map(&map_a, g.act, g.cap, g.p.I, kGM, g.fp8) ||
        !make_map(&map_b, g.w, (int64_t)g.p.E * g.p.N, g.p.I, g.fp8 ? kFN : kGN, g.fp8))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(g.p.out_acc, 0, sizeof(float) * (size_t)g.T * g.p.N, s);
    if (e != cudaSuccess) return e;
    if (g.fp8)
        gemm_combine_fp8_kernel<<<num_sms, kFThreads, kFSmem, s>>>(map_a, map_b, g.p);
    else
        gemm_combine_kernel<<<num_sms, kGThreads, kGSmem, s>>>(map_a, map_b, g.p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n8 = (int64_t)g.T * g.p.N / 8;
    if (n8 > 0) {
        const int grid = (int)((n8 + 255) / 256 < 4 * num_sms ? (n8 + 255) / 256 : 4 * num_sms);
        acc_to_bf16_kernel<<<grid, 256, 0, s>>>(g.p.out_acc, g.out, n8);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace ep
