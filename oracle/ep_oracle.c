/*
 * ep_oracle.c -- CPU oracle for the expert-parallel dispatch/combine path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this file: only the test suite, the smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; the two are compared, never combined.
 *
 * Plain, single-threaded, slow on purpose.  Every function follows the
 * definition the pages give, in the pages' order:
 *
 *   - "lesson14_deepep" (hsthanb4.github.io, practice task, moe_dispatch /
 *     moe_combine): a token is appended to the queue of each of its top-k
 *     experts while looping over tokens i and then over k; combine adds
 *     weight * expert_output back into row i for k = 0..K-1.
 *   - "bowenzhou.top/repos/deepep/01-overview", section 1.1 (EPBuffer.dispatch
 *     signature): expert_alignment, do_expand (one received row per
 *     (token, expert) pair), do_zero_padding; section 1.4 (V1 Buffer.dispatch
 *     signature): num_tokens_per_rank, is_token_in_rank,
 *     num_tokens_per_expert.
 *   - "blog.hotdry.top ... deepep-expert-parallel-alltoall", buffer section:
 *     num_experts % group.size() == 0, i.e. experts split evenly over ranks.
 *   - "2kiu.com/news/5702702" section 2.3 and "m.nlpx.cn/news/135159"
 *     section 4.1: FP8 transport, quantised by the sender with one scaling
 *     factor per block and restored by the receiver.
 *
 * Readings where the pages leave a step open (each listed in the design
 * notes): expert e belongs to rank e / (E/R); rows inside an expert segment
 * are in (token, k) order; a padded segment has ceil(cnt/A)*A rows;
 * num_tokens_per_rank counts distinct tokens; FP8 is OCP E4M3 with one fp32
 * scale per 1x128 block of a token row, amax floored at 1e-4, quantised as
 * e4m3_rne_satfinite(x * (448/amax)) with the dequantisation scale amax/448
 * stored; combine is the exact weighted sum (computed here in fp64); an id
 * of -1 marks a masked top-k slot (no row, no contribution).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_EXPERT 1
#define ORACLE_BAD_ARG 2
#define ORACLE_SLOT_OVERFLOW 3

/* ------------------------------------------------------------------ */
/* Number formats                                                       */
/* ------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE binary32. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a non-negative value below 2^23 to the nearest integer, ties to even. */
static uint32_t round_half_even_u(float q)
{
    float fl = floorf(q);
    float d = q - fl; /* exact: q and fl share the exponent range */
    uint32_t n = (uint32_t)fl;
    if (d > 0.5f) return n + 1;
    if (d < 0.5f) return n;
    return n + (n & 1u);
}

/*
 * OCP 8-bit floating point, E4M3 ("fn") variant: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest
 * finite magnitude 1.75 * 2^8 = 448, subnormals m * 2^-9.  Round to nearest,
 * ties to even; magnitudes at or beyond 448 saturate to 448 ("satfinite").
 */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0f) return (uint8_t)(sign | 0x7E);
    if (a < 0.015625f) {
        /* below 2^-6 the grid is m * 2^-9, m = 0..7; m = 8 is code 0x08 = 2^-6 */
        uint32_t m = round_half_even_u(a * 512.0f);
        return (uint8_t)(sign | m);
    }
    int ex;
    float f = frexpf(a, &ex);              /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;                        /* a = s * 2^e, s in [1, 2)   */
    float q = (f * 2.0f - 1.0f) * 8.0f;    /* fraction of s in units of 1/8 */
    uint32_t m = round_half_even_u(q);
    if (m == 8) { m = 0; e += 1; }
    uint32_t code = ((uint32_t)(e + 7) << 3) | m;
    if (code > 0x7E) code = 0x7E;
    return (uint8_t)(sign | code);
}

void oracle_e4m3_encode_array(int64_t n, const float *v, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------ */
/* Layout                                                               */
/* ------------------------------------------------------------------ */

/* Worst-case number of received rows: every pair plus A-1 padding rows per expert. */
int64_t oracle_capacity_rows(int32_t T, int32_t E, int32_t K, int32_t A)
{
    return (int64_t)T * K + (int64_t)E * (A - 1);
}

/*
 * Layout metadata and the (token, k) -> received-row permutation.
 *
 * topk_idx [T,K] int64, topk_weights [T,K] fp32 or NULL.
 * Outputs: num_tokens_per_expert [E], num_tokens_per_rank [R] (distinct
 * tokens), is_token_in_rank [T,R] bytes, expert_offsets [E+1],
 * rank_offsets [R+1], pos [T,K], and for every received row r < rows:
 * row_src[r] (token or -1 for padding), row_slot[r] (k or -1),
 * row_weight[r] (topk weight or 0; untouched if topk_weights is NULL).
 * An id of -1 marks an unused top-k slot: it gets pos = -1 and no row and
 * is not counted.  Returns ORACLE_BAD_EXPERT if some other id is outside
 * [0, E).
 */
int oracle_layout(int32_t T, int32_t E, int32_t R, int32_t K, int32_t A,
                  const int64_t *topk_idx, const float *topk_weights,
                  int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                  uint8_t *is_token_in_rank, int32_t *expert_offsets,
                  int32_t *rank_offsets, int32_t *pos, int32_t *row_src,
                  int32_t *row_slot, float *row_weight)
{
    if (T < 0 || E <= 0 || R <= 0 || K <= 0 || A <= 0 || E % R != 0)
        return ORACLE_BAD_ARG;
    const int32_t L = E / R; /* local experts per rank */

    /* -1 marks an unused top-k slot (masked: no expert, no row); any other id
       outside [0, E) is an error */
    for (int64_t i = 0; i < (int64_t)T * K; ++i)
        if (topk_idx[i] != -1 && (topk_idx[i] < 0 || topk_idx[i] >= E)) return ORACLE_BAD_EXPERT;

    /* counts per expert: each selected (token, k) pair is one received row */
    for (int32_t e = 0; e < E; ++e) num_tokens_per_expert[e] = 0;
    for (int32_t t = 0; t < T; ++t)
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            if (e >= 0) num_tokens_per_expert[e] += 1;
        }

    /* token membership per rank, and distinct tokens per rank */
    for (int32_t r = 0; r < R; ++r) num_tokens_per_rank[r] = 0;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t r = 0; r < R; ++r) {
            uint8_t in = 0;
            for (int32_t k = 0; k < K; ++k) {
                int64_t e = topk_idx[(int64_t)t * K + k];
                if (e >= 0 && e / L == r) in = 1;
            }
            is_token_in_rank[(int64_t)t * R + r] = in;
            num_tokens_per_rank[r] += in;
        }
    }

    /* padded exclusive offsets; experts of a rank are contiguous */
    expert_offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t c = num_tokens_per_expert[e];
        int32_t padded = ((c + A - 1) / A) * A;
        expert_offsets[e + 1] = expert_offsets[e] + padded;
    }
    for (int32_t r = 0; r <= R; ++r) rank_offsets[r] = expert_offsets[r * L];

    /* dispatch order: loop tokens, then k, append to the expert's queue */
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor) return ORACLE_BAD_ARG;
    for (int32_t e = 0; e < E; ++e) cursor[e] = expert_offsets[e];
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t i = (int64_t)t * K + k;
            int32_t e = (int32_t)topk_idx[i];
            if (e < 0) { pos[i] = -1; continue; }   /* masked slot */
            int32_t r = cursor[e]++;
            pos[i] = r;
            row_src[r] = t;
            row_slot[r] = k;
            if (topk_weights) row_weight[r] = topk_weights[i];
        }
    }
    /* zero padding after each expert's real rows */
    for (int32_t e = 0; e < E; ++e) {
        for (int32_t r = cursor[e]; r < expert_offsets[e + 1]; ++r) {
            row_src[r] = -1;
            row_slot[r] = -1;
            if (topk_weights) row_weight[r] = 0.0f;
        }
    }
    free(cursor);
    return ORACLE_OK;
}

/*
 * Low-latency (static, masked) layout: every expert e owns M fixed slots,
 * received rows e*M .. e*M+M-1, and the per-expert count is the mask a
 * masked grouped GEMM reads ("lesson14_deepep" section 2(1): decode mode is
 * static for CUDA graphs, with pre-allocated buffers and mask marks; section
 * 3: low_latency_dispatch feeds m_grouped_fp8_gemm_nt_masked with a mask).
 * Slots are filled in the same order as the normal layout: tokens, then k.
 *
 * Outputs: recv_count [E] = slots used by expert e (at most M), pos [T,K]
 * = e*M + slot, or -1 for a masked id (-1) or a pair past an expert's M-th.
 * Returns ORACLE_BAD_EXPERT if an id other than -1 is outside [0, E)
 * (outputs unspecified), ORACLE_SLOT_OVERFLOW if some expert was offered
 * more than M pairs (outputs as described), else ORACLE_OK.
 */
int oracle_ll_layout(int32_t T, int32_t E, int32_t K, int32_t M, const int64_t *topk_idx,
                     int32_t *recv_count, int32_t *pos)
{
    if (T < 0 || E <= 0 || K <= 0 || M <= 0) return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < (int64_t)T * K; ++i)
        if (topk_idx[i] != -1 && (topk_idx[i] < 0 || topk_idx[i] >= E)) return ORACLE_BAD_EXPERT;

    int overflow = 0;
    for (int32_t e = 0; e < E; ++e) recv_count[e] = 0;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
            int64_t i = (int64_t)t * K + k;
            int32_t e = (int32_t)topk_idx[i];
            if (e < 0) { pos[i] = -1; continue; }              /* masked slot */
            if (recv_count[e] >= M) { pos[i] = -1; overflow = 1; continue; }
            pos[i] = (int32_t)((int64_t)e * M + recv_count[e]);
            recv_count[e] += 1;
        }
    }
    return overflow ? ORACLE_SLOT_OVERFLOW : ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Dispatch: received row r holds token row_src[r], or zeros           */
/* ------------------------------------------------------------------ */

/*
 * bf16 dispatch for the selected received rows (sel_rows == NULL: rows
 * 0..n_sel-1).  out is [n_sel, H] bf16 bit patterns.
 */
int oracle_dispatch_bf16(int32_t T, int32_t H, int32_t n_sel, const int32_t *sel_rows,
                         const int32_t *row_src, const uint16_t *x, uint16_t *out)
{
    for (int32_t i = 0; i < n_sel; ++i) {
        int32_t r = sel_rows ? sel_rows[i] : i;
        int32_t t = row_src[r];
        uint16_t *dst = out + (int64_t)i * H;
        if (t < 0) {
            memset(dst, 0, sizeof(uint16_t) * (size_t)H);
        } else {
            if (t >= T) return ORACLE_BAD_ARG;
            memcpy(dst, x + (int64_t)t * H, sizeof(uint16_t) * (size_t)H);
        }
    }
    return ORACLE_OK;
}

/* One token row -> e4m3 codes and one dequantisation scale per 128 columns. */
static void quantize_row_e4m3(int32_t H, const uint16_t *xrow, uint8_t *q, float *scale)
{
    for (int32_t b = 0; b < H / 128; ++b) {
        const uint16_t *xb = xrow + b * 128;
        float amax = 0.0f;
        for (int32_t j = 0; j < 128; ++j) amax = fmaxf(amax, fabsf(bf16_bits_to_float(xb[j])));
        float amax_floor = fmaxf(amax, 1e-4f);
        float inv = 448.0f / amax_floor;
        for (int32_t j = 0; j < 128; ++j) {
            float v = bf16_bits_to_float(xb[j]) * inv;
            q[b * 128 + j] = oracle_e4m3_encode(v);
        }
        scale[b] = amax_floor / 448.0f;
    }
}

/*
 * FP8 dispatch for the selected received rows: q [n_sel, H] e4m3 codes,
 * scale [n_sel, H/128] fp32.  Padding rows are code 0x00 with scale 0.
 */
int oracle_dispatch_fp8(int32_t T, int32_t H, int32_t n_sel, const int32_t *sel_rows,
                        const int32_t *row_src, const uint16_t *x, uint8_t *q, float *scale)
{
    if (H % 128 != 0) return ORACLE_BAD_ARG;
    const int32_t nb = H / 128;
    for (int32_t i = 0; i < n_sel; ++i) {
        int32_t r = sel_rows ? sel_rows[i] : i;
        int32_t t = row_src[r];
        uint8_t *qd = q + (int64_t)i * H;
        float *sd = scale + (int64_t)i * nb;
        if (t < 0) {
            memset(qd, 0, (size_t)H);
            for (int32_t b = 0; b < nb; ++b) sd[b] = 0.0f;
        } else {
            if (t >= T) return ORACLE_BAD_ARG;
            quantize_row_e4m3(H, x + (int64_t)t * H, qd, sd);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Combine                                                               */
/* ------------------------------------------------------------------ */

/*
 * out[i, :] = sum_{k=0..K-1} w[t,k] * y[pos[t,k], :]  for t = sel_tokens[i]
 * (sel_tokens == NULL: t = i).  y is [rows, H] bf16, w is [T,K] fp32, the
 * sum is taken in fp64 in k order and returned unrounded.  Masked slots
 * (pos = -1) add nothing.
 */
int oracle_combine(int32_t T, int32_t H, int32_t K, int32_t rows, const int32_t *pos,
                   const uint16_t *y, const float *w, int32_t n_sel,
                   const int32_t *sel_tokens, double *out)
{
    for (int32_t i = 0; i < n_sel; ++i) {
        int32_t t = sel_tokens ? sel_tokens[i] : i;
        if (t < 0 || t >= T) return ORACLE_BAD_ARG;
        double *o = out + (int64_t)i * H;
        for (int32_t h = 0; h < H; ++h) o[h] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int32_t r = pos[(int64_t)t * K + k];
            if (r == -1) continue;                    /* masked slot adds nothing */
            if (r < 0 || r >= rows) return ORACLE_BAD_ARG;
            double wk = (double)w[(int64_t)t * K + k];
            const uint16_t *yr = y + (int64_t)r * H;
            for (int32_t h = 0; h < H; ++h) o[h] += wk * (double)bf16_bits_to_float(yr[h]);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Expert GEMM followed by combine                                      */
/* ------------------------------------------------------------------ */

/*
 * The expert computation that sits between dispatch and combine, for a
 * linear expert map, with combine applied to its output ("lesson14_deepep"
 * practice task: each expert transforms the rows it received, then
 * moe_combine adds weight * expert_output back into the token's row).
 *
 * act [rows, I] bf16 bits: the expert inputs in the received-row layout
 * (row pos[t,k] belongs to pair (t,k)); w [E, N, I] bf16 bits: expert e's
 * matrix, row n holding the weights of output feature n; topk_w [T, K] fp32.
 * For each selected token t (all if sel_tokens is NULL):
 *   out[t, n] = sum_k topk_w[t,k] * sum_i act[pos[t,k], i] * w[e, n, i],
 *   e = topk_idx[t,k], in fp64; pairs with e == -1 (or pos == -1) add nothing.
 */
int oracle_expert_combine(int32_t T, int32_t K, int32_t I, int32_t N, int32_t E, int32_t rows,
                          const int64_t *topk_idx, const int32_t *pos, const uint16_t *act,
                          const uint16_t *w, const float *topk_w, int32_t n_sel,
                          const int32_t *sel_tokens, double *out)
{
    if (T < 0 || K <= 0 || I <= 0 || N <= 0 || E <= 0 || rows < 0) return ORACLE_BAD_ARG;
    for (int32_t j = 0; j < n_sel; ++j) {
        int32_t t = sel_tokens ? sel_tokens[j] : j;
        if (t < 0 || t >= T) return ORACLE_BAD_ARG;
        double *o = out + (int64_t)j * N;
        for (int32_t n = 0; n < N; ++n) o[n] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            int32_t r = pos[(int64_t)t * K + k];
            if (e == -1 || r == -1) continue;
            if (e < 0 || e >= E || r < 0 || r >= rows) return ORACLE_BAD_ARG;
            const uint16_t *a = act + (int64_t)r * I;
            const uint16_t *we = w + (int64_t)e * N * I;
            double wk = (double)topk_w[(int64_t)t * K + k];
            for (int32_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int32_t i = 0; i < I; ++i)
                    acc += (double)bf16_bits_to_float(a[i]) * (double)bf16_bits_to_float(we[(int64_t)n * I + i]);
                o[n] += wk * acc;
            }
        }
    }
    return ORACLE_OK;
}


/*
 * Value of an OCP E4M3 code (sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent 0 is subnormal with step 2^-9; S.1111.111 is NaN; there is
 * no infinity).  Exact in double.
 */
static double e4m3_value(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(8.0 + (double)m, e - 10);   /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }

/*
 * The expert GEMM followed by combine, with FP8 operands: the expert inputs
 * are the E4M3 codes and 1x128 dequantisation scales that the FP8 dispatch
 * writes (a received row restores as q * scale, "2kiu.com/news/5702702"
 * section 2.3), and each expert matrix is E4M3 with one fp32 scale per
 * 128 x 128 block -- the per-block scaling of "m.nlpx.cn/news/135159"
 * section 4.1, consumed by a grouped FP8 GEMM as in "lesson14_deepep"
 * section 3.
 *
 * act_q [rows, I] codes; act_scale: row-major [rows, I/128] when
 * scale_ld == 0, else column-major, scale of (r, b) at act_scale[b * scale_ld + r];
 * w_q [E, N, I] codes; w_scale [E, N/128, I/128].  For each selected token t:
 *   out[t, n] = sum_k topk_w[t,k] * sum_i A[pos[t,k], i] * W_e[n, i],
 *   A[r, i] = q[r, i] * act_scale(r, i/128),
 *   W_e[n, i] = w_q[e, n, i] * w_scale[e, n/128, i/128],
 * e = topk_idx[t,k], in fp64 (every product and partial sum of the tests'
 * inputs is exact there); masked pairs add nothing.
 */
int oracle_expert_combine_fp8(int32_t T, int32_t K, int32_t I, int32_t N, int32_t E, int32_t rows,
                              const int64_t *topk_idx, const int32_t *pos, const uint8_t *act_q,
                              const float *act_scale, int64_t scale_ld, const uint8_t *w_q,
                              const float *w_scale, const float *topk_w, int32_t n_sel,
                              const int32_t *sel_tokens, double *out)
{
    if (T < 0 || K <= 0 || I <= 0 || N <= 0 || E <= 0 || rows < 0) return ORACLE_BAD_ARG;
    if (I % 128 != 0 || N % 128 != 0 || scale_ld < 0 || (scale_ld > 0 && scale_ld < rows)) return ORACLE_BAD_ARG;
    const int32_t IB = I / 128, NB = N / 128;
    double value[256];                    /* e4m3_value of every code, looked up below */
    for (int c = 0; c < 256; ++c) value[c] = e4m3_value((uint8_t)c);
    for (int32_t j = 0; j < n_sel; ++j) {
        int32_t t = sel_tokens ? sel_tokens[j] : j;
        if (t < 0 || t >= T) return ORACLE_BAD_ARG;
        double *o = out + (int64_t)j * N;
        for (int32_t n = 0; n < N; ++n) o[n] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            int32_t r = pos[(int64_t)t * K + k];
            if (e == -1 || r == -1) continue;
            if (e < 0 || e >= E || r < 0 || r >= rows) return ORACLE_BAD_ARG;
            const uint8_t *a = act_q + (int64_t)r * I;
            const uint8_t *we = w_q + (int64_t)e * N * I;
            const float *se = w_scale + (int64_t)e * NB * IB;
            double wk = (double)topk_w[(int64_t)t * K + k];
            for (int32_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int32_t i = 0; i < I; ++i) {
                    int32_t b = i / 128;
                    double sa = scale_ld > 0 ? (double)act_scale[(int64_t)b * scale_ld + r]
                                             : (double)act_scale[(int64_t)r * IB + b];
                    double sw = (double)se[(int64_t)(n / 128) * IB + b];
                    acc += (value[a[i]] * sa) * (value[we[(int64_t)n * I + i]] * sw);
                }
                o[n] += wk * acc;
            }
        }
    }
    return ORACLE_OK;
}
