/*
 * ep_oracle.c -- plain, slow, single-threaded CPU oracle of the MoE
 * expert-parallel dispatch/combine path (layout, dispatch, FP8 dispatch,
 * combine).
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists to check the CUDA library
 * against; only the test suite, the smoke check and the benchmark's CPU
 * baseline may load it.  It shares no code, header, table or helper with
 * the CUDA path.
 *
 * What the path computes comes from the DeepEP pages (the chinainews.com
 * item "DeepSeek releases DeepEP", feature list: all-to-all dispatch and
 * combine for MoE, native FP8 dispatch; the dataforcee.us rewrite, section
 * "Technological Views and Benefits": tokens travel to their experts and
 * the results are merged back; the frogred8 blog, section "Implementation of SMs
 * dedicated to network communication": per-rank senders, up to 8 NVLink
 * peers).  The pages give no formula, so the plain reading used here is:
 *
 *   layout   cnt_e[e]     = #{(t,j) : idx[t,j] == e}
 *            off_e        = exclusive prefix sum of cnt_e (off_e[E] = #valid)
 *            slot_pos[t,j]= off_e[e] + #{(t',j') before (t,j) in token-major
 *                           order with idx[t',j'] == e}   (stable)
 *            recv_src[r]  = token whose copy lands in receive row r
 *            in_rank[t,r] = 1 iff some idx[t,j] lies in rank r's experts
 *                           [r*G, (r+1)*G), G = E/R
 *            cnt_r[r]     = sum_t in_rank[t,r];  off_r = its exclusive scan
 *   dispatch recv[slot_pos[t,j], :] = x[t, :]
 *   FP8      per token t and 128-channel block b:
 *            a = max |x[t, block]| (NaN propagates), a = max(a, 1e-4)
 *            s = a / 448 (fp32, round to nearest)
 *            q = e4m3(x / s) (fp32 quotient, then e4m3 round-to-nearest-even
 *                with saturation to +-448)
 *            q goes to every receive row of t, s to recv_scale[row, b]
 *   combine  out[t,:] = bf16_rne( fma chain over j = 0..k-1 in slot order of
 *                       w[t,j] * y[slot_pos[t,j], :], starting from 0.0f )
 *
 *   aligned layout (receive segments padded for a grouped GEMM whose row
 *            tiles are `align` rows: each expert's segment starts on a
 *            multiple of align)
 *            off_pad      = exclusive prefix sum of ceil(cnt_e / align) * align
 *            slot_pos[t,j]= off_pad[e] + the same stable rank as above
 *            recv_src[r]  = token of row r, -1 for padding rows and past
 *                           off_pad[E], over T*k + E*(align-1) rows
 *   FP8 combine (expert outputs in the FP8 form of dispatch: e4m3 codes and
 *            one fp32 scale per row and 128-channel block)
 *            v = fp32(e4m3 value * scale), rounded to nearest
 *            out[t,:] = bf16_rne( fma chain over j of w[t,j] * v )
 *
 *   replicas (redundant copies of busy experts, EPLB): logical expert e
 *            has n_e = rep_off[e+1] - rep_off[e] physical copies
 *            rep_ids[rep_off[e] .. rep_off[e+1]); the i-th slot choosing e,
 *            counted in token-major order from 0, goes to copy i mod n_e
 *            phys[t,j] = rep_ids[rep_off[e] + (i mod n_e)]
 *
 *   rank layout (the rank-deduplicated form of dispatch: one row per
 *            (token, rank) pair, DeepEP's per-peer sends)
 *            rank_row[t,r] = off_r[r] + #{t' < t : in_rank[t',r]} if
 *                            in_rank[t,r], else -1
 *            rank_src[q]   = token of rank row q (-1 past the last)
 *
 * Slots with idx == -1 are dropped: slot_pos = -1, nothing is written for
 * them and combine skips them.  An id outside [-1, E) is reported
 * (return value EP_ORACLE_ERR_INDEX) and treated like a dropped slot.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math
 * (fmaf is the C library's correctly rounded fused multiply-add).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EP_ORACLE_OK 0
#define EP_ORACLE_ERR_INVALID_ARG 1
#define EP_ORACLE_ERR_INDEX 4

/* ---------------------------------------------------------------- numbers */

/* bf16 -> fp32: a bf16 value is the top half of an fp32 bit pattern. */
float ep_oracle_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even: add half an ulp of the
 * 16 dropped bits (minus one unless the kept lsb is 1) and truncate.  A NaN
 * keeps its sign and top payload bits and is made quiet. */
uint16_t ep_oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* fp32 -> FP8 E4M3 ("e4m3fn": 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite
 * 1.75 * 2^8 = 448, smallest subnormal 2^-9).
 * Round to nearest, ties to even; magnitudes above 448 (infinities too)
 * saturate to +-448; every NaN becomes 0x7f.
 * Written from the format's definition: find the spacing of the
 * representable grid at |v|, round |v| to a multiple of it, re-encode. */
uint8_t ep_oracle_f32_to_e4m3(float v) {
    if (isnan(v))
        return 0x7f;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a > 448.0)
        return sign | 0x7e;
    if (a == 0.0)
        return sign;
    /* binade exponent eb with 2^eb <= a < 2^(eb+1); below the smallest
     * normal 2^-6 the grid keeps the spacing of the first normal binade */
    int fe;
    frexp(a, &fe);                 /* a = m * 2^fe, m in [0.5, 1) */
    int eb = fe - 1;
    if (eb < -6)
        eb = -6;
    const double quantum = ldexp(1.0, eb - 3);
    const double n = nearbyint(a / quantum); /* default mode: ties to even */
    const double r = n * quantum;
    if (r > 448.0)
        return sign | 0x7e;
    if (r < ldexp(1.0, -6))        /* subnormal: r = m * 2^-9, m in 0..7 */
        return sign | (uint8_t)(r / ldexp(1.0, -9));
    frexp(r, &fe);
    const int er = fe - 1;         /* 2^er <= r < 2^(er+1) */
    const int mant = (int)(r / ldexp(1.0, er - 3)) - 8;
    return sign | (uint8_t)(((er + 7) << 3) | mant);
}

/* FP8 E4M3 -> fp32, from the same definition (used by the tests). */
float ep_oracle_e4m3_to_f32(uint8_t q) {
    const int s = q >> 7, e = (q >> 3) & 0xf, m = q & 0x7;
    double v;
    if (e == 0xf && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Element-wise array forms of the two conversions (for the tests). */
void ep_oracle_f32_to_bf16_n(const float *v, long n, uint16_t *out) {
    for (long i = 0; i < n; ++i)
        out[i] = ep_oracle_f32_to_bf16(v[i]);
}

void ep_oracle_f32_to_e4m3_n(const float *v, long n, uint8_t *out) {
    for (long i = 0; i < n; ++i)
        out[i] = ep_oracle_f32_to_e4m3(v[i]);
}

/* ----------------------------------------------------------------- layout */

int ep_oracle_layout(const int64_t *idx, int T, int k, int E, int R,
                     int32_t *cnt_e, int32_t *cnt_r, uint8_t *in_rank,
                     int32_t *off_e, int32_t *off_r, int32_t *slot_pos,
                     int32_t *recv_src) {
    if (T < 0 || k <= 0 || E <= 0 || R <= 0 || E % R != 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    const int G = E / R;
    const long N = (long)T * k;
    int status = EP_ORACLE_OK;

    /* per-expert counts */
    for (int e = 0; e < E; ++e)
        cnt_e[e] = 0;
    for (long i = 0; i < N; ++i) {
        const int64_t e = idx[i];
        if (e == -1)
            continue;
        if (e < -1 || e >= E) {
            status = EP_ORACLE_ERR_INDEX;
            continue;
        }
        cnt_e[e] += 1;
    }

    /* exclusive prefix sum */
    off_e[0] = 0;
    for (int e = 0; e < E; ++e)
        off_e[e + 1] = off_e[e] + cnt_e[e];

    /* stable placement: walk the slots in token-major order and hand each
     * the next free row of its expert */
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    if (!next)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
        next[e] = off_e[e];
    for (long r = 0; r < N; ++r)
        recv_src[r] = -1;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            const long i = (long)t * k + j;
            const int64_t e = idx[i];
            if (e < 0 || e >= E) {
                slot_pos[i] = -1;
                continue;
            }
            const int32_t row = next[e]++;
            slot_pos[i] = row;
            recv_src[row] = t;
        }
    }
    free(next);

    /* token-in-rank mask and per-rank token counts */
    for (int r = 0; r < R; ++r)
        cnt_r[r] = 0;
    for (int t = 0; t < T; ++t) {
        for (int r = 0; r < R; ++r)
            in_rank[(long)t * R + r] = 0;
        for (int j = 0; j < k; ++j) {
            const int64_t e = idx[(long)t * k + j];
            if (e < 0 || e >= E)
                continue;
            in_rank[(long)t * R + e / G] = 1;
        }
        for (int r = 0; r < R; ++r)
            cnt_r[r] += in_rank[(long)t * R + r];
    }
    off_r[0] = 0;
    for (int r = 0; r < R; ++r)
        off_r[r + 1] = off_r[r] + cnt_r[r];
    return status;
}

/* Rank rows from the token-in-rank mask in_rank[T,R]: walk tokens in order,
 * handing each (token, rank) pair the next free row of its rank. */
int ep_oracle_rank_layout(const uint8_t *in_rank, int T, int R, int32_t *cnt_r,
                          int32_t *off_r, int32_t *rank_row, int32_t *rank_src) {
    if (T < 0 || R <= 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int r = 0; r < R; ++r)
        cnt_r[r] = 0;
    for (long i = 0; i < (long)T * R; ++i)
        if (in_rank[i])
            cnt_r[i % R] += 1;
    off_r[0] = 0;
    for (int r = 0; r < R; ++r)
        off_r[r + 1] = off_r[r] + cnt_r[r];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)R);
    if (!next)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int r = 0; r < R; ++r)
        next[r] = off_r[r];
    for (long q = 0; q < (long)T * R; ++q)
        rank_src[q] = -1;
    for (int t = 0; t < T; ++t) {
        for (int r = 0; r < R; ++r) {
            const long i = (long)t * R + r;
            if (!in_rank[i]) {
                rank_row[i] = -1;
                continue;
            }
            rank_row[i] = next[r]++;
            rank_src[rank_row[i]] = t;
        }
    }
    free(next);
    return EP_ORACLE_OK;
}

/* --------------------------------------------------------------- dispatch */

/* Copies token rows to their receive rows.  n_rows bounds the receive
 * buffer; a slot whose row falls outside it is skipped. */
int ep_oracle_dispatch_bf16(const uint16_t *x, int T, int H, int k,
                            const int32_t *slot_pos, long n_rows,
                            uint16_t *recv) {
    if (T < 0 || H <= 0 || k <= 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            const int32_t row = slot_pos[(long)t * k + j];
            if (row < 0 || row >= n_rows)
                continue;
            for (int c = 0; c < H; ++c)
                recv[(long)row * H + c] = x[(long)t * H + c];
        }
    }
    return EP_ORACLE_OK;
}

int ep_oracle_dispatch_fp8(const uint16_t *x, int T, int H, int k,
                           const int32_t *slot_pos, long n_rows,
                           uint8_t *recv_q, float *recv_scale) {
    if (T < 0 || H <= 0 || k <= 0 || H % 128 != 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    const int nb = H / 128;
    uint8_t *q = (uint8_t *)malloc((size_t)H);
    float *s = (float *)malloc(sizeof(float) * (size_t)nb);
    if (!q || !s) {
        free(q);
        free(s);
        return EP_ORACLE_ERR_INVALID_ARG;
    }
    for (int t = 0; t < T; ++t) {
        const uint16_t *xt = x + (long)t * H;
        for (int b = 0; b < nb; ++b) {
            float a = 0.0f;
            for (int c = 128 * b; c < 128 * b + 128; ++c) {
                const float v = fabsf(ep_oracle_bf16_to_f32(xt[c]));
                if (isnan(v) || v > a)
                    a = isnan(a) ? a : v;
            }
            if (a < 1e-4f)
                a = 1e-4f;
            s[b] = a / 448.0f;
            for (int c = 128 * b; c < 128 * b + 128; ++c) {
                const float v = ep_oracle_bf16_to_f32(xt[c]) / s[b];
                q[c] = ep_oracle_f32_to_e4m3(v);
            }
        }
        for (int j = 0; j < k; ++j) {
            const int32_t row = slot_pos[(long)t * k + j];
            if (row < 0 || row >= n_rows)
                continue;
            for (int c = 0; c < H; ++c)
                recv_q[(long)row * H + c] = q[c];
            for (int b = 0; b < nb; ++b)
                recv_scale[(long)row * nb + b] = s[b];
        }
    }
    free(q);
    free(s);
    return EP_ORACLE_OK;
}

/* ---------------------------------------------------------------- combine */

int ep_oracle_combine(const uint16_t *y, long n_rows, int T, int H, int k,
                      const int32_t *slot_pos, const float *w,
                      uint16_t *out) {
    if (T < 0 || H <= 0 || k <= 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    float *acc = (float *)malloc(sizeof(float) * (size_t)H);
    if (!acc)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c)
            acc[c] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int32_t row = slot_pos[(long)t * k + j];
            if (row < 0 || row >= n_rows)
                continue;
            const float wj = w[(long)t * k + j];
            for (int c = 0; c < H; ++c)
                acc[c] = fmaf(wj, ep_oracle_bf16_to_f32(y[(long)row * H + c]),
                              acc[c]);
        }
        for (int c = 0; c < H; ++c)
            out[(long)t * H + c] = ep_oracle_f32_to_bf16(acc[c]);
    }
    free(acc);
    return EP_ORACLE_OK;
}

/* ------------------------------------------------------- aligned layout */

/* Receive rows of the aligned layout: every expert's segment starts on a
 * multiple of `align` rows (its used rows first, in the stable token-major
 * order of ep_oracle_layout, then padding).  recv_src has n_cap =
 * T*k + E*(align-1) entries.  Ids outside [0, E) are dropped (-1). */
int ep_oracle_layout_aligned(const int64_t *idx, int T, int k, int E, int align,
                             int32_t *off_pad, int32_t *slot_pos,
                             int32_t *recv_src) {
    if (T < 0 || k <= 0 || E <= 0 || align <= 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    const long N = (long)T * k;
    const long n_cap = N + (long)E * (align - 1);
    int32_t *cnt = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!cnt || !next) {
        free(cnt);
        free(next);
        return EP_ORACLE_ERR_INVALID_ARG;
    }
    int status = EP_ORACLE_OK;
    for (long i = 0; i < N; ++i) {
        const int64_t e = idx[i];
        if (e >= 0 && e < E)
            cnt[e] += 1;
        else if (e != -1)
            status = EP_ORACLE_ERR_INDEX;
    }
    off_pad[0] = 0;
    for (int e = 0; e < E; ++e) {
        const int32_t padded = (cnt[e] + align - 1) / align * align;
        off_pad[e + 1] = off_pad[e] + padded;
        next[e] = off_pad[e];
    }
    for (long r = 0; r < n_cap; ++r)
        recv_src[r] = -1;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            const long i = (long)t * k + j;
            const int64_t e = idx[i];
            if (e < 0 || e >= E) {
                slot_pos[i] = -1;
                continue;
            }
            const int32_t row = next[e]++;
            slot_pos[i] = row;
            recv_src[row] = t;
        }
    }
    free(cnt);
    free(next);
    return status;
}

/* ---------------------------------------------------------- FP8 combine */

/* Gate-weighted combine of expert outputs given as e4m3 codes yq [n_rows, H]
 * and fp32 scales ys [n_rows, H/128]: each value is decoded and multiplied
 * by its block's scale in fp32, then folded into the fp32 fma chain. */
int ep_oracle_combine_fp8(const uint8_t *yq, const float *ys, long n_rows, int T,
                          int H, int k, const int32_t *slot_pos, const float *w,
                          uint16_t *out) {
    if (T < 0 || H <= 0 || k <= 0 || H % 128 != 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    const int nb = H / 128;
    float *acc = (float *)malloc(sizeof(float) * (size_t)H);
    if (!acc)
        return EP_ORACLE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c)
            acc[c] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int32_t row = slot_pos[(long)t * k + j];
            if (row < 0 || row >= n_rows)
                continue;
            const float wj = w[(long)t * k + j];
            for (int c = 0; c < H; ++c) {
                const float v = ep_oracle_e4m3_to_f32(yq[(long)row * H + c]) *
                                ys[(long)row * nb + c / 128];
                acc[c] = fmaf(wj, v, acc[c]);
            }
        }
        for (int c = 0; c < H; ++c)
            out[(long)t * H + c] = ep_oracle_f32_to_bf16(acc[c]);
    }
    free(acc);
    return EP_ORACLE_OK;
}

/* ------------------------------------------------------------- replicas */

/* Physical expert of every slot: walk the slots in token-major order and
 * deal each logical expert's slots round-robin over its copies.  A dropped
 * slot stays -1; an id outside [-1, E) or an expert without copies is
 * reported and its slot dropped. */
int ep_oracle_map_replicas(const int64_t *idx, int T, int k, int E,
                           const int32_t *rep_off, const int32_t *rep_ids,
                           int32_t *phys) {
    if (T < 0 || k <= 0 || E <= 0)
        return EP_ORACLE_ERR_INVALID_ARG;
    long *seen = (long *)calloc((size_t)E, sizeof(long));
    if (!seen)
        return EP_ORACLE_ERR_INVALID_ARG;
    int status = EP_ORACLE_OK;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            const long i = (long)t * k + j;
            const int64_t e = idx[i];
            phys[i] = -1;
            if (e == -1)
                continue;
            if (e < -1 || e >= E || rep_off[e + 1] <= rep_off[e]) {
                status = EP_ORACLE_ERR_INDEX;
                continue;
            }
            const long n = rep_off[e + 1] - rep_off[e];
            phys[i] = rep_ids[rep_off[e] + seen[e] % n];
            seen[e] += 1;
        }
    }
    free(seen);
    return status;
}
