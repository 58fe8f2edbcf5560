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
// Phases, separated by two bounded grid-wide waits:
//   1. chunk histogram of experts (shared-memory atomics: counts only) and of
//      distinct tokens per rank; is_token_in_rank rows.
//   2. exclusive scan of every histogram column over the chunks
//      (one warp per column), column totals.
//   3. padded exclusive scan over experts; stable ranks inside the chunk with
//      __match_any_sync + popc(lanemask_lt) per warp and a per-warp prefix
//      table in shared memory, so no atomic ever decides a position.
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

// Grid-wide wait with a %globaltimer limit.  Returns false (and sets
// EP_DEV_WAIT_TIMEOUT) if the other CTAs did not all arrive in time; the
// caller then returns without touching memory again.
__device__ bool grid_wait(const LayoutParams &p, int *s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        GridBarrier *b = p.barrier;
        const unsigned int expected = (unsigned int)(p.G + p.barrier_extra);
        const unsigned int gen = ld_acquire_u32(&b->gen);
        __threadfence();
        const unsigned int arrived = atomicAdd(&b->count, 1u) + 1u;
        int ok = 1;
        if (arrived == expected) {
            atomicExch(&b->count, 0u);
            __threadfence();
            atomicAdd(&b->gen, 1u);
        } else {
            const unsigned long long t0 = globaltimer_ns();
            while (ld_acquire_u32(&b->gen) == gen) {
                if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                    ok = 0;
                    atomicOr(p.status, EP_DEV_WAIT_TIMEOUT);
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

__device__ __forceinline__ bool valid_expert(int64_t e, int E) { return e >= 0 && e < E; }

__global__ void __launch_bounds__(kLayoutThreads, 1) layout_kernel(LayoutParams p) {
    extern __shared__ int32_t smem[];
    const int E = p.E, R = p.R, K = p.K, L = p.L;
    const int ncols = E + R;
    int32_t *s_hist = smem;              // [E+R]  chunk histogram, later column totals
    int32_t *s_base = s_hist + ncols;    // [E]    next free row per expert for this chunk
    int32_t *s_eoff = s_base + E;        // [E+1]  padded expert offsets
    int32_t *s_warp = s_eoff + (E + 1);  // [kLayoutWarps][E] per-warp prefix table
    __shared__ int32_t s_tmp[kLayoutWarps + 1];
    __shared__ int s_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const int t_begin = min(p.T, c * p.tokens_per_chunk);
    const int t_end = min(p.T, t_begin + p.tokens_per_chunk);
    const int64_t p_begin = (int64_t)t_begin * K, p_end = (int64_t)t_end * K;

    // ---- phase 1: chunk histograms ------------------------------------------
    for (int i = tid; i < ncols; i += kLayoutThreads) s_hist[i] = 0;
    __syncthreads();
    for (int64_t q = p_begin + tid; q < p_end; q += kLayoutThreads) {
        const int64_t e = p.topk_idx[q];
        if (valid_expert(e, E))
            atomicAdd(&s_hist[e], 1);
        else
            atomicOr(p.status, EP_DEV_BAD_EXPERT);
    }
    for (int t = t_begin + tid; t < t_end; t += kLayoutThreads) {
        const int64_t *row = p.topk_idx + (int64_t)t * K;
        if (R <= 64) {
            unsigned long long mask = 0;
            for (int k = 0; k < K; ++k) {
                const int64_t e = row[k];
                if (!valid_expert(e, E)) continue;
                const int r = (int)(e / L);
                if (!((mask >> r) & 1ull)) {
                    mask |= 1ull << r;
                    atomicAdd(&s_hist[E + r], 1);
                }
            }
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
            for (int k = 0; k < K; ++k) {
                const int64_t e = row[k];
                if (!valid_expert(e, E)) continue;
                const int r = (int)(e / L);
                bool dup = false;
                for (int k2 = 0; k2 < k; ++k2) {
                    const int64_t e2 = row[k2];
                    if (valid_expert(e2, E) && (int)(e2 / L) == r) dup = true;
                }
                if (!dup) atomicAdd(&s_hist[E + r], 1);
            }
            if (p.u_in_rank) {
                uint8_t *dst = p.u_in_rank + (int64_t)t * R;
                for (int r = 0; r < R; ++r) dst[r] = 0;
                for (int k = 0; k < K; ++k) {
                    const int64_t e = row[k];
                    if (valid_expert(e, E)) dst[e / L] = 1;
                }
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < ncols; i += kLayoutThreads)
        p.chunk_counts[(int64_t)c * ncols + i] = s_hist[i];

    if (!grid_wait(p, &s_flag)) return;

    // ---- phase 2: exclusive scan of each column over the chunks -------------
    for (int j = c * kLayoutWarps + warp; j < ncols; j += p.G * kLayoutWarps) {
        int carry = 0;
        for (int cb = 0; cb < p.G; cb += 32) {
            const int cc = cb + lane;
            const int v = cc < p.G ? __ldcg(&p.chunk_counts[(int64_t)cc * ncols + j]) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            if (cc < p.G) p.chunk_counts[(int64_t)cc * ncols + j] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) p.col_total[j] = carry;
    }

    if (!grid_wait(p, &s_flag)) return;

    // ---- phase 3: offsets and stable ranks ----------------------------------
    for (int i = tid; i < ncols; i += kLayoutThreads) s_hist[i] = __ldcg(&p.col_total[i]);
    __syncthreads();
    for (int e = tid; e < E; e += kLayoutThreads) s_eoff[e] = (s_hist[e] + p.A - 1) / p.A * p.A;
    __syncthreads();
    const int rows = block_exclusive_scan(s_eoff, E, s_tmp);
    if (tid == 0) s_eoff[E] = rows;
    for (int e = tid; e < E; e += kLayoutThreads)
        s_base[e] = s_eoff[e] + __ldcg(&p.chunk_counts[(int64_t)c * ncols + e]);
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
    // padding rows of experts c, c+G, ...
    for (int e = c; e < E; e += p.G) {
        const int r0 = s_eoff[e] + s_hist[e], r1 = s_eoff[e + 1];
        for (int r = r0 + tid; r < r1; r += kLayoutThreads) {
            p.row_src[r] = -1;
            p.row_slot[r] = -1;
            if (p.topk_weights) p.row_weight[r] = 0.0f;
        }
    }

    // stable ranks, one tile of kLayoutThreads consecutive pairs at a time
    for (int64_t tile = p_begin; tile < p_end; tile += kLayoutThreads) {
        for (int i = tid; i < kLayoutWarps * E; i += kLayoutThreads) s_warp[i] = 0;
        __syncthreads();
        const int64_t q = tile + tid;
        const bool in_range = q < p_end;
        int e = -1;
        if (in_range) {
            const int64_t v = p.topk_idx[q];
            e = valid_expert(v, E) ? (int)v : -1;
        }
        const unsigned int peers = __match_any_sync(0xffffffffu, e);
        const int lrank = __popc(peers & lanemask_lt());
        if (e >= 0 && lrank == 0) s_warp[warp * E + e] = __popc(peers);
        __syncthreads();
        for (int e2 = tid; e2 < E; e2 += kLayoutThreads) {
            int run = s_base[e2];
#pragma unroll
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
                if (p.topk_weights) p.row_weight[dst] = p.topk_weights[q];
            } else {
                p.pos[q] = -1;
            }
        }
        __syncthreads();
    }
}

}  // namespace

size_t layout_smem_bytes(int E, int R) {
    return sizeof(int32_t) * ((size_t)(E + R) + E + (E + 1) + (size_t)kLayoutWarps * E);
}

const void *layout_kernel_ptr() { return reinterpret_cast<const void *>(&layout_kernel); }

cudaError_t launch_layout(const LayoutParams &p, size_t smem, cudaStream_t s) {
    LayoutParams args = p;
    void *kargs[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(&layout_kernel), dim3(p.G),
                                       dim3(kLayoutThreads), kargs, smem, s);
}

}  // namespace ep
