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
// Two kernels compute the same result.  layout_cluster_kernel, used
// whenever a CTA can hold its share (at most 8192 pairs per CTA, 16 CTAs),
// is one thread-block cluster: every warp ranks a contiguous range of pairs
// while it loads them, and the CTAs exchange their histograms through
// distributed shared memory, so there is no global scratch and no polled
// barrier.  layout_kernel, the fallback for larger batches, is a cooperative
// grid:
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
#include <cooperative_groups.h>

#include "ep_internal.cuh"

#ifndef EP_LAYOUT_TRIGGER_LATE
#define EP_LAYOUT_TRIGGER_LATE 0   // 1: the cluster kernel lets a dependent launch start after its id
                                   // loads (measured the same as at its start)
#endif

namespace ep {

namespace {

// Grid-wide wait with a %globaltimer limit.  The arrival counter only grows:
// after `epoch` completed waits it holds epoch * G, and this wait ends when it
// reaches (epoch + 1) * G, so no reset is needed between launches.  Each CTA
// reads the epoch before it arrives, and CTA 0 advances it once every CTA has
// arrived (so every CTA has read it): the target comes from the device, and a
// launch replayed from a CUDA graph finds the right one.  Returns false (and
// sets EP_DEV_WAIT_TIMEOUT) if the other CTAs did not all arrive in time; the
// caller then returns without touching memory again (ep_clear_status resets
// the counter and the epoch).
__device__ bool grid_wait(const LayoutParams &p, int *s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int *count = &p.barrier->count;
        const unsigned int epoch = ld_acquire_u32(&p.barrier->epoch);
        const unsigned int target = (epoch + 1) * (unsigned int)(p.G + p.barrier_extra);
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
        if (ok && blockIdx.x == 0) atomicExch(&p.barrier->epoch, epoch + 1);
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

__device__ __forceinline__ bool valid_expert(int64_t e, int E) { return e >= 0 && e < E; }

// is_token_in_rank row of one token from its rank mask (R <= 64), four
// bytes per store when the row is 4-byte aligned.
__device__ __forceinline__ void write_in_rank_row(uint8_t *dst, int R, unsigned long long mask) {
    if ((R & 3) == 0 && ((reinterpret_cast<uintptr_t>(dst) & 3) == 0)) {
        for (int r = 0; r < R; r += 4) {
            const unsigned int bits = (unsigned int)(mask >> r) & 0xfu;
            const unsigned int word = (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 |
                                      ((bits >> 3) & 1u) << 24;
            *reinterpret_cast<unsigned int *>(dst + r) = word;
        }
    } else {
        for (int r = 0; r < R; ++r) dst[r] = (uint8_t)((mask >> r) & 1ull);
    }
}



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
    pdl_launch_dependents();   // a dispatch launched next may start its set-up now
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
    // padding rows of experts c, c+G, ...: one warp per expert, its lanes
    // over consecutive rows
    for (int e = c + G * warp; e < E; e += G * kLayoutWarps) {
        const int r0 = s_eoff[e] + s_hist[e], r1 = s_eoff[e + 1];
        for (int r = r0 + (tid & 31); r < r1; r += 32) {
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

// ---------------------------------------------------------------------------
// Cluster layout.  CTA c of the cluster takes tokens
// [c*tokens_per_chunk, (c+1)*tokens_per_chunk); inside it, warp w takes a
// contiguous range of ppw pairs (a multiple of 32, at most
// kClusterMaxSteps*32) and walks it 32 pairs at a time in (token, k) order.
// Per step, each lane finds the lanes with the same expert from ballots over
// the id bits; its rank inside the warp's range is the warp's running count
// of that expert (a private shared-memory row) plus the peers below it.
// The rows of counts then become exclusive prefixes over the warps, the CTA
// histograms are read across the cluster (distributed shared memory) for
// the totals and the pairs of earlier CTAs, and a pair's row is
// offset + earlier CTAs + earlier warps + rank in warp.  A CTA's rows of one
// expert are consecutive, so the row-indexed outputs are staged in shared
// memory in the CTA's own row order and written out segment by segment:
// the stores coalesce instead of scattering one sector per pair.
// ---------------------------------------------------------------------------
constexpr int kClusterMaxSteps = 4;
constexpr int kClusterMaxPairs = kLayoutThreads * kClusterMaxSteps;   // pairs per CTA

// Exclusive scans of a[0..n) and b[0..n) in shared memory, in place, in one
// pass; returns both totals.  Caller must have synchronised after writing.
__device__ int2 block_exclusive_scan2(int32_t *a, int32_t *b, int n, int32_t *s_tmp /*[2*(kLayoutWarps+1)]*/) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kLayoutThreads - 1) / kLayoutThreads;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int sa = 0, sb = 0;
    for (int i = lo; i < hi; ++i) {
        sa += a[i];
        sb += b[i];
    }
    int ia = sa, ib = sb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int va = __shfl_up_sync(0xffffffffu, ia, o), vb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += va;
            ib += vb;
        }
    }
    int32_t *ta = s_tmp, *tb = s_tmp + (kLayoutWarps + 1);
    if (lane == 31) {
        ta[warp] = ia;
        tb[warp] = ib;
    }
    __syncthreads();
    if (warp == 0) {
        const int va = lane < kLayoutWarps ? ta[lane] : 0, vb = lane < kLayoutWarps ? tb[lane] : 0;
        int xa = va, xb = vb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ua = __shfl_up_sync(0xffffffffu, xa, o), ub = __shfl_up_sync(0xffffffffu, xb, o);
            if (lane >= o) {
                xa += ua;
                xb += ub;
            }
        }
        if (lane < kLayoutWarps) {
            ta[lane] = xa - va;
            tb[lane] = xb - vb;
        }
        if (lane == 31) {
            ta[kLayoutWarps] = xa;
            tb[kLayoutWarps] = xb;
        }
    }
    __syncthreads();
    int ra = ta[warp] + ia - sa, rb = tb[warp] + ib - sb;
    for (int i = lo; i < hi; ++i) {
        const int va = a[i], vb = b[i];
        a[i] = ra;
        b[i] = rb;
        ra += va;
        rb += vb;
    }
    const int2 tot = make_int2(ta[kLayoutWarps], tb[kLayoutWarps]);
    __syncthreads();
    return tot;
}

// Expert (low 16 bits, -1: none) of a pair's packed shared-memory entry.
__device__ __forceinline__ int cl_expert(int er) { return (int)(short)(er & 0xffff); }

__global__ void __launch_bounds__(kLayoutThreads, 1) layout_cluster_kernel(LayoutParams p) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    extern __shared__ int32_t smem[];
    const int E = p.E, R = p.R, K = p.K, L = p.L;
    const int ncols = E + R, ES = E + 1;            // ES: padded row stride (no bank conflicts)
    int32_t *s_cnt = smem;                          // [kLayoutWarps][ES] per-warp counts, then prefixes
    int32_t *s_hist = s_cnt + kLayoutWarps * ES;    // [E+R] this CTA's counts (read by the cluster)
    int32_t *s_tot = s_hist + ncols;                // [E+R] cluster totals
    int32_t *s_before = s_tot + ncols;              // [E]   pairs of expert e in earlier CTAs
    int32_t *s_eoff = s_before + E;                 // [E+1] padded expert offsets
    int32_t *s_loff = s_eoff + (E + 1);             // [E+1] this CTA's rows: exclusive offsets per expert
    int32_t *s_er = s_loff + (E + 1);               // [steps][kLayoutThreads] pair: expert | rank << 16
    int32_t *s_qe = s_er + kClusterMaxPairs;        // [pairs] in this CTA's row order: pair | expert << 16
    float *s_wp = reinterpret_cast<float *>(s_qe + kClusterMaxPairs);        // [pairs] weight, pair order
    int16_t *s_ep = reinterpret_cast<int16_t *>(s_wp + kClusterMaxPairs);  // [pairs] expert (-1: none), pair order
    int16_t *s_rk = s_ep + kClusterMaxPairs;                                // [E] rank of expert e
    __shared__ int32_t s_tmp[2 * (kLayoutWarps + 1)];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#if !EP_LAYOUT_TRIGGER_LATE
    pdl_launch_dependents();   // a dispatch launched next may start its set-up now
#endif
    const int t_begin = min(p.T, c * p.tokens_per_chunk);
    const int t_end = min(p.T, t_begin + p.tokens_per_chunk);
    const int64_t p_begin = (int64_t)t_begin * K;
    const int npairs = (int)((int64_t)t_end * K - p_begin);
    const int ppw = (npairs + kLayoutThreads - 1) / kLayoutThreads * 32;   // pairs per warp
    const int steps = ppw / 32;
    const int w_lo = warp * ppw, w_hi = min(npairs, w_lo + ppw);          // this warp's local pairs

    // every id and weight of this warp's range is requested before any is
    // used; the shared-memory set-up runs while they are in flight
    int64_t v_id[kClusterMaxSteps];
    float v_w[kClusterMaxSteps];
#pragma unroll
    for (int j = 0; j < kClusterMaxSteps; ++j) {
        const int i = w_lo + j * 32 + lane;
        const bool in = j < steps && i < w_hi;
        v_id[j] = in ? __ldg(p.topk_idx + p_begin + i) : (int64_t)-1;
        v_w[j] = (in && p.topk_weights) ? __ldg(p.topk_weights + p_begin + i) : 0.0f;
    }
    for (int i = tid; i < kLayoutWarps * ES; i += kLayoutThreads) s_cnt[i] = 0;
    for (int i = tid; i < ncols; i += kLayoutThreads) s_hist[i] = 0;
    for (int e = tid; e < E; e += kLayoutThreads) s_rk[e] = (int16_t)(e / L);
#pragma unroll
    for (int j = 0; j < kClusterMaxSteps; ++j) {
        if (j < steps) {
            const int i = w_lo + j * 32 + lane;
            const int64_t v = v_id[j];
            const int e = valid_expert(v, E) ? (int)v : -1;
            if (i < w_hi && e < 0 && v != -1) atomicOr(p.status, EP_DEV_BAD_EXPERT);   // -1: masked slot
            s_er[j * kLayoutThreads + tid] = e & 0xffff;
            if (i < w_hi) {
                s_ep[i] = (int16_t)e;
                s_wp[i] = v_w[j];
            }
        }
    }
#if EP_LAYOUT_TRIGGER_LATE
    pdl_launch_dependents();   // after this CTA's only DRAM reads
#endif
    __syncthreads();
    int32_t *wrow = s_cnt + warp * ES;
#pragma unroll 1
    for (int j = 0; j < steps; ++j) {
        const int er = s_er[j * kLayoutThreads + tid];
        const int e = cl_expert(er);
        unsigned int peers = __ballot_sync(0xffffffffu, e >= 0);
        if (e < 0) peers = ~peers;
        for (int b = 0; b < p.id_bits; ++b) {
            const int bit = (e >> b) & 1;
            const unsigned int bal = __ballot_sync(0xffffffffu, bit);
            peers &= bit ? bal : ~bal;
        }
        const int lrank = __popc(peers & lanemask_lt());
        const int base = e >= 0 ? wrow[e] : 0;
        __syncwarp();
        if (e >= 0 && lrank == 0) wrow[e] = base + __popc(peers);
        __syncwarp();
        s_er[j * kLayoutThreads + tid] = er | ((base + lrank) << 16);
    }
    __syncthreads();

    // exclusive prefix of each expert's counts over the warps; P lanes share
    // one expert, each summing 32/P rows, with a shuffle scan across them
    {
        int P = 1;
        while (P < 32 && 2 * P * E <= kLayoutThreads) P <<= 1;
        const int e = tid / P, part = tid % P, rows = kLayoutWarps / P;
        const bool act = e < E;
        int local = 0;
        if (act) {
#pragma unroll 8
            for (int w = part * rows; w < (part + 1) * rows; ++w) local += s_cnt[w * ES + e];
        }
        int incl = local;
        for (int o = 1; o < P; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o, P);
            if (part >= o) incl += v;
        }
        if (act) {
            int run = incl - local;
            for (int w = part * rows; w < (part + 1) * rows; ++w) {
                const int v = s_cnt[w * ES + e];
                s_cnt[w * ES + e] = run;
                run += v;
            }
            if (part == P - 1) s_hist[e] = run;
        }
    }
    // distinct tokens per rank and is_token_in_rank rows, from the staged ids
    if (R <= 64 && K <= 32 && (K & (K - 1)) == 0) {
        // a token's K pairs are K consecutive lanes of one warp: each lane
        // contributes its pair's rank bit and a shuffle OR gives the token's
        // mask.  Lane j of a token's group then writes words j, j+K, ... of
        // its is_token_in_rank row and counts ranks j, j+K, ... : the counts
        // of the warp's tokens are summed by shuffles and added to the
        // histogram by the group's first K lanes, one address per lane.
        const int span = (npairs + 31) / 32 * 32;
        const int j = lane & (K - 1);
        const bool row_words = p.u_in_rank && (R & 3) == 0 && (reinterpret_cast<uintptr_t>(p.u_in_rank) & 3) == 0;
        for (int i = tid; i < span; i += kLayoutThreads) {
            const bool tok = i < npairs;
            const int e = tok ? s_ep[i] : -1;
            const int r = e >= 0 ? s_rk[e] : -1;
            unsigned int lo = (r >= 0 && r < 32) ? 1u << r : 0u;
            unsigned int hi = r >= 32 ? 1u << (r - 32) : 0u;
            for (int o = 1; o < K; o <<= 1) {
                lo |= __shfl_xor_sync(0xffffffffu, lo, o);
                hi |= __shfl_xor_sync(0xffffffffu, hi, o);
            }
            const unsigned long long mask = ((unsigned long long)hi << 32) | lo;
            for (int rb = 0; rb < R; rb += K) {
                const int rr = rb + j;
                int c = (tok && rr < R) ? (int)((mask >> rr) & 1ull) : 0;
                for (int o = K; o < 32; o <<= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
                if (lane < K && rr < R && c) atomicAdd(&s_hist[E + rr], c);
            }
            if (tok && p.u_in_rank) {
                uint8_t *row = p.u_in_rank + (int64_t)(t_begin + i / K) * R;
                if (row_words) {
                    for (int w = j; w < R / 4; w += K) {
                        const unsigned int bits = (unsigned int)(mask >> (4 * w)) & 0xfu;
                        reinterpret_cast<unsigned int *>(row)[w] = (bits & 1u) | ((bits >> 1) & 1u) << 8 |
                                                                  ((bits >> 2) & 1u) << 16 | ((bits >> 3) & 1u) << 24;
                    }
                } else {
                    for (int q = j; q < R; q += K) row[q] = (uint8_t)((mask >> q) & 1ull);
                }
            }
        }
    } else {
        for (int t = t_begin + tid; t < t_end; t += kLayoutThreads) {
            const int i0 = (t - t_begin) * K;
            if (R <= 64) {
                unsigned long long mask = 0;
                for (int k = 0; k < K; ++k) {
                    const int e = s_ep[i0 + k];
                    if (e >= 0) mask |= 1ull << s_rk[e];
                }
                for (unsigned long long m = mask; m; m &= m - 1)
                    atomicAdd(&s_hist[E + __ffsll((long long)m) - 1], 1);
                if (p.u_in_rank) write_in_rank_row(p.u_in_rank + (int64_t)t * R, R, mask);
            } else {
                // more than 64 ranks: distinct ranks by pairwise comparison
                uint8_t *dst = p.u_in_rank ? p.u_in_rank + (int64_t)t * R : nullptr;
                if (dst)
                    for (int r = 0; r < R; ++r) dst[r] = 0;
                for (int k = 0; k < K; ++k) {
                    const int e = s_ep[i0 + k];
                    if (e < 0) continue;
                    const int r = s_rk[e];
                    bool dup = false;
                    for (int k2 = 0; k2 < k; ++k2) {
                        const int e2 = s_ep[i0 + k2];
                        if (e2 >= 0 && s_rk[e2] == r) dup = true;
                    }
                    if (!dup) atomicAdd(&s_hist[E + r], 1);
                    if (dst) dst[r] = 1;
                }
            }
        }
    }
    if (C > 1) {
        // every CTA's histogram complete and visible to the cluster
        cluster.sync();
        for (int j = tid; j < ncols; j += kLayoutThreads) {
            int v[16];                              // all remote reads in flight together
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) v[cc] = cc < C ? *cluster.map_shared_rank(s_hist + j, cc) : 0;
            int tot = 0, before = 0;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
                tot += v[cc];
                before += cc < c ? v[cc] : 0;
            }
            s_tot[j] = tot;
            if (j < E) s_before[j] = before;
        }
        // this CTA is done reading the others' shared memory; it must not exit
        // before they are done reading its own (waited for at the end)
        cluster.barrier_arrive();
    } else {
        // one CTA (small batches): its histogram is the total, no cluster exchange
        __syncthreads();
        for (int j = tid; j < ncols; j += kLayoutThreads) {
            s_tot[j] = s_hist[j];
            if (j < E) s_before[j] = 0;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kLayoutThreads) {
        s_eoff[e] = (s_tot[e] + p.A - 1) / p.A * p.A;
        s_loff[e] = s_hist[e];
    }
    __syncthreads();
    const int2 totals = block_exclusive_scan2(s_eoff, s_loff, E, s_tmp);
    if (tid == 0) {
        s_eoff[E] = totals.x;
        s_loff[E] = totals.y;
    }
    __syncthreads();

    // pos in pair order; each pair's entry staged at its row in this CTA's order
#pragma unroll 1
    for (int j = 0; j < steps; ++j) {
        const int i = w_lo + j * 32 + lane;
        if (i < w_hi) {
            const int er = s_er[j * kLayoutThreads + tid];
            const int e = cl_expert(er);
            if (e >= 0) {
                const int within = wrow[e] + (er >> 16);   // rank among this CTA's pairs of e
                p.pos[p_begin + i] = s_eoff[e] + s_before[e] + within;
                s_qe[s_loff[e] + within] = i | (e << 16);
            } else {
                p.pos[p_begin + i] = -1;
            }
        }
    }
    __syncthreads();
    for (int lr = tid; lr < s_loff[E]; lr += kLayoutThreads) {
        const int qe = s_qe[lr];
        const int i = qe & 0xffff, e = qe >> 16;
        const int dst = s_eoff[e] + s_before[e] + (lr - s_loff[e]);
        const int64_t q = p_begin + i;
        const int t = (int)(q / K);
        p.row_src[dst] = t;
        p.row_slot[dst] = (int)(q - (int64_t)t * K);
        if (p.topk_weights) p.row_weight[dst] = s_wp[i];
    }
    if (c == 0) {
        for (int e = tid; e < E; e += kLayoutThreads) {
            p.cnt[e] = s_tot[e];
            if (p.u_cnt) p.u_cnt[e] = s_tot[e];
        }
        for (int r = tid; r < R; r += kLayoutThreads) {
            p.rank_tok[r] = s_tot[E + r];
            if (p.u_rank_tok) p.u_rank_tok[r] = s_tot[E + r];
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
    // padding rows of experts c, c+C, ...: one warp per expert, its lanes
    // over consecutive rows
    for (int e = c + C * warp; e < E; e += C * kLayoutWarps) {
        const int r0 = s_eoff[e] + s_tot[e], r1 = s_eoff[e + 1];
        for (int r = r0 + lane; r < r1; r += 32) {
            p.row_src[r] = -1;
            p.row_slot[r] = -1;
            if (p.topk_weights) p.row_weight[r] = 0.0f;
        }
    }
    if (C > 1) cluster.barrier_wait();
}

size_t cluster_smem_bytes(int E, int R) {
    return sizeof(int32_t) * ((size_t)kLayoutWarps * (E + 1) + 2 * (size_t)(E + R) + E + 2 * (size_t)(E + 1) +
                              3 * (size_t)kClusterMaxPairs) +
           sizeof(int16_t) * ((size_t)kClusterMaxPairs + E);
}

}  // namespace

size_t layout_smem_bytes(int E, int R) {
    return sizeof(int32_t) * ((size_t)(E + R) + E + (E + 1) + (size_t)kLayoutWarps * E + kLayoutThreads);
}

const void *layout_kernel_ptr() { return reinterpret_cast<const void *>(&layout_kernel); }

// Per device, once: kernel attributes (dynamic shared memory for the
// largest supported E and R, clusters of 16) and the largest cluster size
// that can be resident with one 1024-thread CTA per SM.
static int g_max_cluster[kMaxDevices];

cudaError_t layout_prepare(int device) {
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    if (__atomic_load_n(&g_max_cluster[device], __ATOMIC_ACQUIRE) > 0) return cudaSuccess;
    const void *coop = reinterpret_cast<const void *>(&layout_kernel);
    const void *clus = reinterpret_cast<const void *>(&layout_cluster_kernel);
    cudaError_t e = cudaFuncSetAttribute(coop, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)layout_smem_bytes(kMaxExperts, kMaxExperts));
    if (e != cudaSuccess) return e;
    const size_t csmem = cluster_smem_bytes(kMaxExperts, kMaxExperts);
    e = cudaFuncSetAttribute(clus, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem);
    if (e != cudaSuccess) return e;
    int best = 1;
    if (cudaFuncSetAttribute(clus, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        for (int cs = 16; cs >= 2 && best == 1; cs /= 2) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(cs);
            cfg.blockDim = dim3(kLayoutThreads);
            cfg.dynamicSmemBytes = csmem;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = cs;
            attr.val.clusterDim.y = 1;
            attr.val.clusterDim.z = 1;
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, clus, &cfg) == cudaSuccess && n >= 1) best = cs;
        }
    }
    cudaGetLastError();   // a refused size query leaves no sticky error behind
    __atomic_store_n(&g_max_cluster[device], best, __ATOMIC_RELEASE);
    return cudaSuccess;
}

LayoutPlan plan_layout(int device, int T, int E, int R, int K, int num_sms) {
    LayoutPlan pl{};
    const int64_t pairs = (int64_t)T * K;
    const int cmax = (device >= 0 && device < kMaxDevices) ? __atomic_load_n(&g_max_cluster[device], __ATOMIC_ACQUIRE) : 0;
    if (cmax >= 1) {
        // about kClusterPairsTarget pairs per CTA, at most kClusterMaxPairs
        int C = (int)((pairs + kClusterPairsTarget - 1) / kClusterPairsTarget);
        C = C < 1 ? 1 : C;
        while (C < cmax && (int64_t)((T + C - 1) / C) * K > kClusterMaxPairs) ++C;
        if (C > cmax) C = cmax;
        // cluster sizes that are powers of two schedule best; round up
        int Cp = 1;
        while (Cp < C) Cp <<= 1;
        if (Cp <= cmax) C = Cp;
        const int tpc = T > 0 ? (T + C - 1) / C : 1;
        if ((int64_t)tpc * K <= kClusterMaxPairs) {
            pl.cluster = true;
            pl.G = C;
            pl.tokens_per_chunk = tpc;
            pl.smem = cluster_smem_bytes(E, R);
            return pl;
        }
    }
    int64_t G = (pairs + kLayoutPairsPerCta - 1) / kLayoutPairsPerCta;
    G = G < 1 ? 1 : (G > num_sms ? num_sms : G);   // one CTA per SM at most
    const int tpc = T > 0 ? (int)((T + G - 1) / G) : 1;
    G = T > 0 ? (T + tpc - 1) / tpc : 1;
    pl.cluster = false;
    pl.G = (int)G;
    pl.tokens_per_chunk = tpc;
    pl.smem = layout_smem_bytes(E, R);
    return pl;
}

cudaError_t launch_layout(const LayoutParams &p, const LayoutPlan &pl, cudaStream_t s) {
    if (pl.cluster) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pl.G);
        cfg.blockDim = dim3(kLayoutThreads);
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = s;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = pl.G;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, layout_cluster_kernel, p);
    }
    if (p.G == 1) {   // a single CTA never waits on another: plain launch
        layout_kernel<<<1, kLayoutThreads, pl.smem, s>>>(p);
        return cudaGetLastError();
    }
    LayoutParams args = p;
    void *kargs[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(&layout_kernel), dim3(p.G),
                                       dim3(kLayoutThreads), kargs, pl.smem, s);
}

}  // namespace ep
