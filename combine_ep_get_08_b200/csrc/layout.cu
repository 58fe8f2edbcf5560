// layout.cu -- routing layout for dispatch/combine (sm_100a).
//
// From topk_idx [T, K] this computes, in one cooperative launch of G CTAs
// (one chunk of consecutive tokens per CTA):
//   num_tokens_per_expert, distinct tokens per rank, is_token_in_rank,
//   padded expert offsets (expert_alignment), rank offsets, and the stable
//   permutation pos[t, k] -> received row with its inverse row_src/row_slot
//   (and row_weight).
// Rows of an expert are in (token, k) order, the order in which the
// lesson14_deepep practice task appends tokens to each expert's queue;
// per-expert segments are padded to a multiple of expert_alignment
// (EPBuffer.dispatch arguments expert_alignment / do_zero_padding,
// bowenzhou.top "deepep/01-overview" section 1.1).
//
// Phases, separated by one bounded grid-wide wait (none when G == 1):
//   1. chunk histogram of experts (shared-memory atomics decide counts only)
//      and of distinct tokens per rank; is_token_in_rank rows.  The
//      histogram is published column-major, chunk_counts[j][c].
//   2. every CTA sums each column twice over the chunks -- all chunks
//      (totals) and chunks before its own (its starting rank inside each
//      expert) -- with independent 16-byte loads; then the padded exclusive
//      scan over experts.
//   3. stable ranks inside the chunk: each lane finds the lanes of its warp
//      with the same expert from ballots over the id bits, and a per-warp
//      prefix table in shared memory orders the warps, so no atomic ever
//      decides a position.
#include "ep_internal.cuh"

namespace ep {

namespace {

// Exclusive scan of a[0..n) in shared memory, in place; returns the total.
// Caller must have synchronised after writing a[].
__device__ int block_exclusive_scan(int32_t *a, int n, int32_t *s_tmp /*[kLayoutWarps+1]*/) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kLayoutThreads - 1) / kLayoutThreads;
    const int b = min(n, tid * per), e = min(n, b + per);
    int sum = 0;
    for (int i = b; i < e; ++i) sum += a[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kLayoutWarps ? s_tmp[lane] : 0;
        int iv = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, iv, o);
            if (lane >= o) iv += u;
        }
        if (lane < kLayoutWarps) s_tmp[lane] = iv - v;
        if (lane == 31) s_tmp[kLayoutWarps] = iv;
    }
    __syncthreads();
    int run = s_tmp[warp] + incl - sum;
    for (int i = b; i < e; ++i) {
        int v = a[i];
        a[i] = run;
        run += v;
    }
    const int total = s_tmp[kLayoutWarps];
    __syncthreads();
    return total;
}

// Grid-wide wait with a %globaltimer limit.  The arrival counter only grows:
// launch number `epoch` (1, 2, ...) waits until it reaches epoch * G, so no
// reset is needed between launches.  Returns false (and sets
// EP_DEV_WAIT_TIMEOUT) if the other CTAs did not all arrive in time; the
// caller then returns without touching memory again.
__device__ bool grid_wait(const LayoutParams &p, int *s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int *count = &p.barrier->count;
        const unsigned int target = p.epoch * (unsigned int)(p.G + p.barrier_extra);
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" : : "l"(count) : "memory");
        int ok = 1;
        if ((int)(ld_acquire_u32(count) - target) < 0) {
            const unsigned long long t0 = globaltimer_ns();
            while ((int)(ld_acquire_u32(count) - target) < 0) {
                if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                    ok = 0;
                    atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                    break;
                }
            }
        }
        __threadfence();
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

__device__ __forceinline__ bool valid_expert(int64_t e, int E) { return e >= 0 && e < E; }

// Loads up to 8 consecutive expert ids of one token (all loads issued
// before any is used); missing entries read as -1.
__device__ __forceinline__ void load_ids8(const int64_t *row, int k0, int K, int64_t (&ev)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) ev[j] = (k0 + j < K) ? __ldg(row + k0 + j) : -1;
}

__global__ void __launch_bounds__(kLayoutThreads, 1) layout_kernel(LayoutParams p) {
    extern __shared__ int32_t smem[];
    const int E = p.E, R = p.R, K = p.K, L = p.L, G = p.G;
    const int ncols = E + R;
    int32_t *s_hist = smem;              // [E+R]  chunk histogram, later column totals
    int32_t *s_base = s_hist + ncols;    // [E]    next free row per expert for this chunk
    int32_t *s_eoff = s_base + E;        // [E+1]  padded expert offsets
    int32_t *s_warp = s_eoff + (E + 1);  // [kLayoutWarps][E] per-warp prefix table
    int32_t *s_ids = s_warp + kLayoutWarps * E;   // [kLayoutThreads] expert ids of a one-tile chunk
    __shared__ int32_t s_tmp[kLayoutWarps + 1];
    __shared__ int s_flag;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int c = blockIdx.x;
    const int t_begin = min(p.T, c * p.tokens_per_chunk);
    const int t_end = min(p.T, t_begin + p.tokens_per_chunk);
    const int64_t p_begin = (int64_t)t_begin * K, p_end = (int64_t)t_end * K;

    // ---- phase 1: chunk histograms ------------------------------------------
    // A chunk of at most kLayoutThreads pairs (the usual case) is read once:
    // thread i keeps pair i's id and weight in registers for phase 3 and
    // stages the id in shared memory for the per-token pass.
    const bool one_tile = p_end - p_begin <= kLayoutThreads;
    int my_e = -1;
    float my_w = 0.0f;
    for (int i = tid; i < ncols; i += kLayoutThreads) s_hist[i] = 0;
    if (one_tile && tid < p_end - p_begin) {
        const int64_t v = __ldg(p.topk_idx + p_begin + tid);
        my_e = valid_expert(v, E) ? (int)v : -1;
        if (p.topk_weights) my_w = __ldg(p.topk_weights + p_begin + tid);
        if (my_e < 0 && v != -1) atomicOr(p.status, EP_DEV_BAD_EXPERT);   // -1: masked slot
        s_ids[tid] = my_e;
    }
    __syncthreads();
    if (one_tile) {
        if (my_e >= 0) atomicAdd(&s_hist[my_e], 1);
    } else {
        for (int64_t q = p_begin + tid; q < p_end; q += kLayoutThreads) {
            const int64_t e = __ldg(p.topk_idx + q);
            if (valid_expert(e, E))
                atomicAdd(&s_hist[e], 1);
            else if (e != -1)
                atomicOr(p.status, EP_DEV_BAD_EXPERT);
        }
    }
    for (int t = t_begin + tid; t < t_end; t += kLayoutThreads) {
        const int64_t *row = p.topk_idx + (int64_t)t * K;
        const int *srow = s_ids + (t - t_begin) * K;   // valid when one_tile
        if (R <= 64) {
            unsigned long long mask = 0;
            if (one_tile) {
                for (int k = 0; k < K; ++k)
                    if (srow[k] >= 0) mask |= 1ull << (srow[k] / L);
            } else {
                for (int k0 = 0; k0 < K; k0 += 8) {
                    int64_t ev[8];
                    load_ids8(row, k0, K, ev);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (valid_expert(ev[j], E)) mask |= 1ull << (int)(ev[j] / L);
                }
            }
            for (unsigned long long m = mask; m; m &= m - 1) atomicAdd(&s_hist[E + __ffsll((long long)m) - 1], 1);
            if (p.u_in_rank) {
                uint8_t *dst = p.u_in_rank + (int64_t)t * R;
                if ((R & 3) == 0 && ((reinterpret_cast<uintptr_t>(dst) & 3) == 0)) {
                    for (int r = 0; r < R; r += 4) {
                        const unsigned int bits = (unsigned int)(mask >> r) & 0xfu;
                        const unsigned int word = (bits & 1u) | ((bits >> 1) & 1u) << 8 |
                                                  ((bits >> 2) & 1u) << 16 | ((bits >> 3) & 1u) << 24;
                        *reinterpret_cast<unsigned int *>(dst + r) = word;
                    }
                } else {
                    for (int r = 0; r < R; ++r) dst[r] = (uint8_t)((mask >> r) & 1ull);
                }
            }
        } else {
            // more than 64 ranks: distinct ranks by pairwise comparison
            for (int k = 0; k < K; ++k) {
                const int64_t e = __ldg(row + k);
                if (!valid_expert(e, E)) continue;
                const int r = (int)(e / L);
                bool dup = false;
                for (int k2 = 0; k2 < k; ++k2) {
                    const int64_t e2 = __ldg(row + k2);
                    if (valid_expert(e2, E) && (int)(e2 / L) == r) dup = true;
                }
                if (!dup) atomicAdd(&s_hist[E + r], 1);
            }
            if (p.u_in_rank) {
                uint8_t *dst = p.u_in_rank + (int64_t)t * R;
                for (int r = 0; r < R; ++r) dst[r] = 0;
                for (int k = 0; k < K; ++k) {
                    const int64_t e = __ldg(row + k);
                    if (valid_expert(e, E)) dst[e / L] = 1;
                }
            }
        }
    }
    __syncthreads();

    // ---- phase 2: column sums over chunks -----------------------------------
    if (G == 1) {
        // one chunk: its histogram is the total and it starts every expert
        for (int e = tid; e < E; e += kLayoutThreads) s_base[e] = 0;
    } else {
        const int Gp = p.G_stride;   // row stride of chunk_counts (multiple of 4; tail stays 0)
        for (int j = tid; j < ncols; j += kLayoutThreads) p.chunk_counts[(int64_t)j * Gp + c] = s_hist[j];
        if (!grid_wait(p, &s_flag)) return;
        for (int j = tid; j < ncols; j += kLayoutThreads) s_hist[j] = 0;
        for (int e = tid; e < E; e += kLayoutThreads) s_base[e] = 0;
        __syncthreads();
        // A segment of S lanes (S = Gq rounded up to a power of two, at most
        // 32) owns one column per pass: lane l of the segment reads quads
        // l, l + S, ... of the column's chunk counts (16-byte loads), the
        // segment adds them with xor shuffles and its first lane writes the
        // total and the chunk's prefix.  Loads of up to kBatch quads per
        // thread are issued before any is used.
        const int Gq = Gp / 4;
        int S = 1;
        while (S < Gq && S < 32) S <<= 1;
        const int qpl = (Gq + S - 1) / S;             // quads per lane per column
        const int cols_per_pass = kLayoutThreads / S;
        const int passes = (ncols + cols_per_pass - 1) / cols_per_pass;
        const int seg = tid / S, sl = tid % S;
        const int4 *cc4 = reinterpret_cast<const int4 *>(p.chunk_counts);
        constexpr int kBatch = 4;
        const int pass_per_batch = qpl >= kBatch ? 1 : kBatch / qpl;
        for (int pb = 0; pb < passes; pb += pass_per_batch) {
            const int np = min(pass_per_batch, passes - pb);
            for (int m0 = 0; m0 < qpl; m0 += kBatch) {     // more than kBatch quads per lane: chunks of kBatch
                const int nm = min(kBatch, qpl - m0);
                int4 v[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int pi = u / nm, m = m0 + u % nm;
                    const int j = seg + (pb + pi) * cols_per_pass;
                    const int q = sl + m * S;
                    v[u] = (pi < np && j < ncols && q < Gq) ? __ldcg(cc4 + (int64_t)j * Gq + q)
                                                            : make_int4(0, 0, 0, 0);
                }
                for (int pi = 0; pi < np; ++pi) {
                    const int j = seg + (pb + pi) * cols_per_pass;
                    int tot = 0, before = 0;
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        if (u / nm != pi) continue;
                        const int c0 = 4 * (sl + (m0 + u % nm) * S);
                        tot += v[u].x + v[u].y + v[u].z + v[u].w;
                        before += (c0 < c ? v[u].x : 0) + (c0 + 1 < c ? v[u].y : 0) +
                                  (c0 + 2 < c ? v[u].z : 0) + (c0 + 3 < c ? v[u].w : 0);
                    }
                    for (int o = S / 2; o >= 1; o >>= 1) {
                        tot += __shfl_xor_sync(0xffffffffu, tot, o);
                        before += __shfl_xor_sync(0xffffffffu, before, o);
                    }
                    if (sl == 0 && j < ncols) {
                        s_hist[j] += tot;
                        if (j < E) s_base[j] += before;
                    }
                }
            }
        }
    }
    __syncthreads();
    // padded exclusive scan over experts, then each expert's first row for
    // this chunk
    for (int e = tid; e < E; e += kLayoutThreads) s_eoff[e] = (s_hist[e] + p.A - 1) / p.A * p.A;
    __syncthreads();
    const int rows = block_exclusive_scan(s_eoff, E, s_tmp);
    if (tid == 0) s_eoff[E] = rows;
    for (int e = tid; e < E; e += kLayoutThreads) s_base[e] += s_eoff[e];
    __syncthreads();

    if (c == 0) {
        for (int e = tid; e < E; e += kLayoutThreads) {
            p.cnt[e] = s_hist[e];
            if (p.u_cnt) p.u_cnt[e] = s_hist[e];
        }
        for (int r = tid; r < R; r += kLayoutThreads) {
            p.rank_tok[r] = s_hist[E + r];
            if (p.u_rank_tok) p.u_rank_tok[r] = s_hist[E + r];
        }
        for (int e = tid; e <= E; e += kLayoutThreads) {
            p.eoff[e] = s_eoff[e];
            if (p.u_eoff) p.u_eoff[e] = s_eoff[e];
        }
        for (int r = tid; r <= R; r += kLayoutThreads) {
            p.roff[r] = s_eoff[r * L];
            if (p.u_roff) p.u_roff[r] = s_eoff[r * L];
        }
    }
    // padding rows of experts c, c+G, ..., one expert per thread
    for (int e = c + G * tid; e < E; e += G * kLayoutThreads) {
        const int r0 = s_eoff[e] + s_hist[e], r1 = s_eoff[e + 1];
        for (int r = r0; r < r1; ++r) {
            p.row_src[r] = -1;
            p.row_slot[r] = -1;
            if (p.topk_weights) p.row_weight[r] = 0.0f;
        }
    }

    // ---- phase 3: stable ranks, one tile of kLayoutThreads pairs at a time --
    for (int64_t tile = p_begin; tile < p_end; tile += kLayoutThreads) {
        for (int i = tid; i < kLayoutWarps * E; i += kLayoutThreads) s_warp[i] = 0;
        const int64_t q = tile + tid;
        const bool in_range = q < p_end;
        int e = my_e;
        float wq = my_w;
        if (!one_tile) {
            e = -1;
            if (in_range) {
                const int64_t v = __ldg(p.topk_idx + q);
                e = valid_expert(v, E) ? (int)v : -1;
                if (p.topk_weights) wq = __ldg(p.topk_weights + q);
            }
        }
        __syncthreads();
        // lanes of the warp holding the same expert: one ballot per bit of the
        // id (ceil(log2 E) ballots) plus one for validity
        unsigned int peers = __ballot_sync(0xffffffffu, e >= 0);
        if (e < 0) peers = ~peers;
        for (int b = 0; b < p.id_bits; ++b) {
            const int bit = (e >> b) & 1;
            const unsigned int bal = __ballot_sync(0xffffffffu, bit);
            peers &= bit ? bal : ~bal;
        }
        const int lrank = __popc(peers & lanemask_lt());
        const int wcount = __popc(peers);
        if (e >= 0 && lrank == 0) s_warp[warp * E + e] = wcount;
        __syncthreads();
        for (int e2 = tid; e2 < E; e2 += kLayoutThreads) {
            int run = s_base[e2];
#pragma unroll 8
            for (int w = 0; w < kLayoutWarps; ++w) {
                const int v = s_warp[w * E + e2];
                s_warp[w * E + e2] = run;
                run += v;
            }
            s_base[e2] = run;
        }
        __syncthreads();
        if (in_range) {
            if (e >= 0) {
                const int dst = s_warp[warp * E + e] + lrank;
                const int t = (int)(q / K);
                p.pos[q] = dst;
                p.row_src[dst] = t;
                p.row_slot[dst] = (int)(q - (int64_t)t * K);
                if (p.topk_weights) p.row_weight[dst] = wq;
            } else {
                p.pos[q] = -1;
            }
        }
        __syncthreads();
    }
}

}  // namespace

size_t layout_smem_bytes(int E, int R) {
    return sizeof(int32_t) * ((size_t)(E + R) + E + (E + 1) + (size_t)kLayoutWarps * E + kLayoutThreads);
}

const void *layout_kernel_ptr() { return reinterpret_cast<const void *>(&layout_kernel); }

cudaError_t launch_layout(const LayoutParams &p, size_t smem, cudaStream_t s) {
    if (p.G == 1) {   // a single CTA never waits on another: plain launch
        layout_kernel<<<1, kLayoutThreads, smem, s>>>(p);
        return cudaGetLastError();
    }
    LayoutParams args = p;
    void *kargs[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(&layout_kernel), dim3(p.G),
                                       dim3(kLayoutThreads), kargs, smem, s);
}

}  // namespace ep
