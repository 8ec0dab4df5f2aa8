/*
 * CPU oracle for the single-GPU MoE FFN layer: route -> dispatch -> expert
 * SwiGLU FFN -> combine.
 *
 * TEST INFRASTRUCTURE. Plain, slow, obviously correct loops that restate the
 * definition of each step. Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm load this file's library; the product path
 * never does. It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (page title, section):
 *  "MoE 专家并行的 All-to-All 通信瓶颈：专家越多推理延迟为何反而上升"
 *       §All-to-All 分发与回收的机制 (dataflow flowchart: route Top-K, pack by
 *       destination card, group by expert, grouped GEMM, weighted merge back to
 *       token order), §专家越多，通信为什么越重 (E/W experts per card, even
 *       placement, per-card send volume N*K*d*b/W).
 *  "MoE 推理服务工程真相 2026 ..." §2.2 Expert Capacity Factor (tokens above
 *       an expert's capacity are dropped, router output set to zero) and the
 *       moe_dispatch pseudo-code of §2.3 (bincount of expert ids, overflow mask).
 *  "MoE Inference Communication" §DeepSpeed-MoE › MoE 计算核优化 (top-k,
 *       cumsum, scatter; dense token->expert mapping table), §ExFlow 跨层专家
 *       亲和性 (conditional routing between consecutive layers), §Aurora 定理
 *       4.2 (traffic matrix D).
 *  "MoE 推理服务工程真相 2026 ..." §6.3 通信压缩 (the token payload of the all-to-all in FP8
 *       instead of BF16).
 * Readings where the pages are silent (all fixed by the workload statement):
 *  softmax over the K selected logits; ties to the lowest expert index; logits
 *  accumulated in fp32 by one fused multiply-add per input element, i
 *  ascending, then + bias; capacity C = ceil(cf*N*K/E) computed in double;
 *  first-come drop in token-major (t, k) order; a dropped slot contributes 0
 *  and the others keep their weights; SwiGLU experts y = W2 (silu(W1 x) * W3 x)
 *  without biases; experts in contiguous blocks of E/W per rank; tokens in
 *  contiguous shards of N/W per home rank.
 *
 * Floating point: logits in fp32 (the precision the selection is defined in);
 * expert FFN, gate weights and combine in fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

static float bf16_to_float(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Router projection [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制,
 * node B; MoE Inference Communication, §Aurora, gate term G_i]. logits[t][e] = (sum_i x[t][i] * Wr[e][i]) + bias[e], the sum taken
 * as one fmaf per i in ascending order starting from +0.0f. */
EXPORT void orc_router_logits(int64_t N, int64_t d, int64_t E, const uint16_t *x,
                              const float *w_router, const float *bias, float *logits)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int64_t i = 0; i < d; ++i)
                acc = fmaf(bf16_to_float(x[t * d + i]), w_router[e * d + i], acc);
            if (bias)
                acc = acc + bias[e];
            logits[t * E + e] = acc;
        }
    }
}

/* Top-K selection and gate weights [MoE 专家并行的 All-to-All 通信瓶颈, §一个反直觉的
 * 扩容结果 (Top-K experts per token); MoE Inference Communication, §MoE 计算核优化 (top-k)].
 * The K largest logits, larger value first, equal values ordered by lower expert index. Weights: softmax over the K
 * selected logits, in fp64, stored as fp32. Returns the number of tokens that
 * have a non-finite logit (their result is unspecified). */
EXPORT int64_t orc_topk(int64_t N, int64_t E, int64_t K, const float *logits,
                        int32_t *topk_idx, float *topk_w)
{
    int64_t nonfinite = 0;
    char *chosen = (char *)malloc((size_t)E);
    double *ex = (double *)malloc((size_t)K * sizeof(double));
    for (int64_t t = 0; t < N; ++t) {
        const float *l = logits + t * E;
        int bad = 0;
        for (int64_t e = 0; e < E; ++e) {
            chosen[e] = 0;
            if (!isfinite(l[e]))
                bad = 1;
        }
        nonfinite += bad;
        for (int64_t k = 0; k < K; ++k) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (chosen[e])
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            chosen[best] = 1;
            topk_idx[t * K + k] = (int32_t)best;
        }
        double top = (double)l[topk_idx[t * K]];
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            ex[k] = exp((double)l[topk_idx[t * K + k]] - top);
            sum += ex[k];
        }
        for (int64_t k = 0; k < K; ++k)
            topk_w[t * K + k] = (float)(ex[k] / sum);
    }
    free(ex);
    free(chosen);
    return nonfinite;
}

/* Expert capacity [MoE 推理服务工程真相 2026, §2.2]: C = ceil(cf * N * K / E), in double.
 * cf <= 0 means dropless; then C = N * K, which no expert can exceed (each token picks K
 * distinct experts, so an expert receives at most N). */
EXPORT int64_t orc_capacity(int64_t N, int64_t E, int64_t K, float cf)
{
    if (!(cf > 0.0f))
        return N * K;
    return (int64_t)ceil((double)cf * (double)N * (double)K / (double)E);
}

/* Position of each assignment in its expert's sequence, walking the N*K assignments in
 * priority order: token-major (order 0: a = t*K + k in increasing a) or slot-major
 * (order 1: every token's slot 0, tokens ascending, then every token's slot 1, ...).
 * Only assignments with expert[a] >= 0 take part; start[e] is where expert e's count
 * begins (0 for a first pass). */
static void walk_positions(int64_t N, int64_t E, int64_t K, int64_t order,
                           const int64_t *expert, const int64_t *start, int64_t *pos,
                           int64_t *total)
{
    for (int64_t e = 0; e < E; ++e)
        total[e] = start ? start[e] : 0;
    for (int64_t idx = 0; idx < N * K; ++idx) {
        int64_t a = order == 0 ? idx : (idx % N) * K + idx / N;
        int64_t e = expert[a];
        if (e < 0)
            continue;
        pos[a] = total[e];
        total[e] += 1;
    }
}

/* Dispatch bookkeeping [MoE 推理服务工程真相 2026, §2.3 pseudo-code (bincount, overflow
 * mask, remapping of overflowed assignments); §2.2 (capacity, expert drop); §4.3 (token
 * drop: re-route to the next-best expert); MoE Inference Communication, §MoE 计算核优化
 * (cumsum, scatter, mapping table); MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与
 * 回收的机制 (pack by destination card)].
 *
 * First pass: pos0[a] = number of earlier assignments (in priority order) to the
 * same expert; the assignment is kept iff pos0 < C. demand counts[e] = all
 * assignments routed to e.
 *
 * With reroute: an expert is full when counts[e] >= C. Each assignment that
 * overflowed (pos0 >= C) moves to its token's best-ranked expert (larger logit
 * first, ties to the lower index) that is neither one of the token's K routed
 * experts, nor full, nor already taken by an earlier overflowed slot (in k order)
 * of the same token; none such: it stays dropped. The moved assignments then take
 * positions at their new expert after all of its first-pass assignments, in the
 * same priority order, and are kept iff that position < C. They keep their gate
 * weight. One round: a moved assignment that does not fit is dropped.
 *
 * Results: expert_of[a] = the expert whose row a uses, -1 if dropped.
 * kept[e] = rows of expert e; offsets = exclusive scan of kept (E+1 entries);
 * row_of[a] = offsets[expert_of[a]] + position, or -1; assign_of_row its inverse.
 *
 * Virtual ranks: expert e lives on rank e / (E/W); token t's home is t / (N/W).
 * D[i][j] counts rows from home i at experts on rank j. The packed buffer holds
 * blocks (i, j) in row-major order; inside a block, expert by expert in
 * increasing e, the rows of that expert whose token's home is i, in row order.
 * pk_off is the exclusive scan of D (W*W+1 entries) and packed_row_of[a] the row
 * of assignment a there (-1 if dropped).
 *
 * stats[0] R (rows), [1] dropped = N*K - R, [2] rows with rank(e) != home(t),
 * [3] distinct (t, rank) pairs with rank != home(t) over the rows (what a
 * deduplicating exchange would send), [4] experts with rows, [5] max kept[e],
 * [6] min kept[e], [7] C, [8] rows at a re-routed expert. */
EXPORT void orc_dispatch(int64_t N, int64_t E, int64_t K, int64_t W, int64_t C, int64_t order,
                         int64_t reroute, const float *logits, const int32_t *topk_idx,
                         int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of,
                         int32_t *assign_of_row, int32_t *expert_of, int64_t *D,
                         int64_t *pk_off, int32_t *packed_row_of, int64_t *stats)
{
    int64_t e_per = E / W, n_per = N / W;
    int64_t NK = N * K;
    int64_t *route = (int64_t *)malloc((size_t)NK * sizeof(int64_t));
    int64_t *pos = (int64_t *)malloc((size_t)NK * sizeof(int64_t));
    int64_t *moved = (int64_t *)malloc((size_t)NK * sizeof(int64_t));
    int64_t *pos1 = (int64_t *)malloc((size_t)NK * sizeof(int64_t));
    int64_t *demand = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *total = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    char *taken = (char *)malloc((size_t)E);

    for (int64_t a = 0; a < NK; ++a) {
        route[a] = topk_idx[a];
        moved[a] = -1;
    }
    walk_positions(N, E, K, order, route, NULL, pos, demand);

    int64_t n_moved = 0;
    if (reroute) {
        for (int64_t t = 0; t < N; ++t) {
            memset(taken, 0, (size_t)E);
            for (int64_t k = 0; k < K; ++k)
                taken[topk_idx[t * K + k]] = 1;
            for (int64_t k = 0; k < K; ++k) {
                int64_t a = t * K + k;
                if (pos[a] < C)
                    continue;
                const float *l = logits + t * E;
                int64_t best = -1;
                for (int64_t e = 0; e < E; ++e) {
                    if (taken[e] || demand[e] >= C)
                        continue;
                    if (best < 0 || l[e] > l[best])
                        best = e;
                }
                if (best >= 0) {
                    taken[best] = 1;
                    moved[a] = best;
                }
            }
        }
        /* second pass starts after each expert's first-pass assignments */
        walk_positions(N, E, K, order, moved, demand, pos1, total);
    }

    for (int64_t a = 0; a < NK; ++a) {
        if (pos[a] < C) {
            expert_of[a] = (int32_t)route[a];
        } else if (moved[a] >= 0 && pos1[a] < C) {
            expert_of[a] = (int32_t)moved[a];
            pos[a] = pos1[a];
            n_moved += 1;
        } else {
            expert_of[a] = -1;
        }
    }

    for (int64_t e = 0; e < E; ++e) {
        counts[e] = (int32_t)demand[e];
        kept[e] = 0;
    }
    for (int64_t a = 0; a < NK; ++a)
        if (expert_of[a] >= 0)
            kept[expert_of[a]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + kept[e];
    for (int64_t i = 0; i < W * W; ++i)
        D[i] = 0;
    int64_t R = 0, cross = 0;
    for (int64_t a = 0; a < NK; ++a) {
        int64_t e = expert_of[a];
        if (e < 0) {
            row_of[a] = -1;
            continue;
        }
        int64_t r = offsets[e] + pos[a];
        row_of[a] = (int32_t)r;
        assign_of_row[r] = (int32_t)a;
        int64_t i = (a / K) / n_per, j = e / e_per;
        D[i * W + j] += 1;
        if (i != j)
            cross += 1;
        R += 1;
    }
    pk_off[0] = 0;
    for (int64_t b = 0; b < W * W; ++b)
        pk_off[b + 1] = pk_off[b] + D[b];

    for (int64_t a = 0; a < NK; ++a)
        packed_row_of[a] = -1;
    int64_t next = 0;
    for (int64_t i = 0; i < W; ++i)
        for (int64_t j = 0; j < W; ++j)
            for (int64_t e = j * e_per; e < (j + 1) * e_per; ++e)
                for (int64_t r = offsets[e]; r < offsets[e + 1]; ++r) {
                    int64_t a = assign_of_row[r];
                    if ((a / K) / n_per == i)
                        packed_row_of[a] = (int32_t)(next++);
                }

    /* distinct destination ranks per token, excluding the home rank */
    int64_t dedup = 0;
    char *rank_seen = (char *)malloc((size_t)W);
    for (int64_t t = 0; t < N; ++t) {
        memset(rank_seen, 0, (size_t)W);
        for (int64_t k = 0; k < K; ++k) {
            int64_t e = expert_of[t * K + k];
            if (e < 0)
                continue;
            int64_t j = e / e_per;
            if (j != t / n_per && !rank_seen[j]) {
                rank_seen[j] = 1;
                dedup += 1;
            }
        }
    }
    int64_t active = 0, mx = 0, mn = -1;
    for (int64_t e = 0; e < E; ++e) {
        if (kept[e] > 0)
            active += 1;
        if (kept[e] > mx)
            mx = kept[e];
        if (mn < 0 || kept[e] < mn)
            mn = kept[e];
    }
    stats[0] = R;
    stats[1] = NK - R;
    stats[2] = cross;
    stats[3] = dedup;
    stats[4] = active;
    stats[5] = mx;
    stats[6] = mn;
    stats[7] = C;
    stats[8] = n_moved;
    free(rank_seen);
    free(taken);
    free(total);
    free(demand);
    free(pos1);
    free(moved);
    free(pos);
    free(route);
}

/* Without re-routing: the priority order alone decides. */
EXPORT void orc_positions_ordered(int64_t N, int64_t E, int64_t K, int64_t W, int64_t C,
                                  int64_t order, const int32_t *topk_idx, int32_t *counts,
                                  int32_t *kept, int32_t *offsets, int32_t *row_of,
                                  int32_t *assign_of_row, int64_t *D, int64_t *pk_off,
                                  int32_t *packed_row_of, int64_t *stats)
{
    int32_t *expert_of = (int32_t *)malloc((size_t)(N * K) * sizeof(int32_t));
    int64_t st[9];
    orc_dispatch(N, E, K, W, C, order, 0, NULL, topk_idx, counts, kept, offsets, row_of,
                 assign_of_row, expert_of, D, pk_off, packed_row_of, st);
    for (int i = 0; i < 8; ++i)
        stats[i] = st[i];
    free(expert_of);
}

/* Token-major priority without re-routing (the default reading). */
EXPORT void orc_positions(int64_t N, int64_t E, int64_t K, int64_t W, int64_t C,
                          const int32_t *topk_idx, int32_t *counts, int32_t *kept,
                          int32_t *offsets, int32_t *row_of, int32_t *assign_of_row,
                          int64_t *D, int64_t *pk_off, int32_t *packed_row_of,
                          int64_t *stats)
{
    orc_positions_ordered(N, E, K, W, C, 0, topk_idx, counts, kept, offsets, row_of,
                          assign_of_row, D, pk_off, packed_row_of, stats);
}

/* Expert FFN for a list of rows [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与
 * 回收的机制, node F: each expert's tokens through its own FFN]. Row r holds the hidden state of token
 * row_token[r] for expert row_expert[r]:
 *   g = W1[e] x, u = W3[e] x, h = g * sigmoid(g) * u, y = W2[e] h,
 * all in fp64 from the bf16 inputs. W1, W3 are [E][f][d]; W2 is [E][d][f].
 * h_out (nullable) receives h [nrows][f]; y_out receives y [nrows][d]. */
EXPORT void orc_expert_rows(int64_t nrows, const int32_t *row_token, const int32_t *row_expert,
                            int64_t d, int64_t f, const uint16_t *x, const uint16_t *w1,
                            const uint16_t *w3, const uint16_t *w2, double *h_out, double *y_out)
{
#pragma omp parallel
    {
        double *xr = (double *)malloc((size_t)d * sizeof(double));
        double *h = (double *)malloc((size_t)f * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = row_token[r], e = row_expert[r];
            for (int64_t i = 0; i < d; ++i)
                xr[i] = (double)bf16_to_float(x[t * d + i]);
            for (int64_t j = 0; j < f; ++j) {
                const uint16_t *a = w1 + (e * f + j) * d;
                const uint16_t *b = w3 + (e * f + j) * d;
                double g = 0.0, u = 0.0;
                for (int64_t i = 0; i < d; ++i) {
                    g += xr[i] * (double)bf16_to_float(a[i]);
                    u += xr[i] * (double)bf16_to_float(b[i]);
                }
                h[j] = g / (1.0 + exp(-g)) * u;
                if (h_out)
                    h_out[r * f + j] = h[j];
            }
            for (int64_t i = 0; i < d; ++i) {
                const uint16_t *c = w2 + (e * d + i) * f;
                double y = 0.0;
                for (int64_t j = 0; j < f; ++j)
                    y += h[j] * (double)bf16_to_float(c[j]);
                y_out[r * d + i] = y;
            }
        }
        free(h);
        free(xr);
    }
}

/* Weighted combine [MoE 专家并行的 All-to-All 通信瓶颈, §All-to-All 分发与回收的机制,
 * node I: weighted merge back to the original token order; MoE 推理服务工程真相 2026, §2.2:
 * a dropped slot's router output is zero]. out[t] = sum over kept slots k, in k order, of w[t][k] * y[row], where
 * y_of_slot[(t*K+k)*d ...] holds the expert output of slot (t, k). */
EXPORT void orc_combine(int64_t N, int64_t K, int64_t d, const int32_t *row_of,
                        const float *topk_w, const double *y_of_slot, double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int64_t i = 0; i < d; ++i)
            out[t * d + i] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int64_t a = t * K + k;
            if (row_of[a] < 0)
                continue;
            double w = (double)topk_w[a];
            for (int64_t i = 0; i < d; ++i)
                out[t * d + i] += w * y_of_slot[a * d + i];
        }
    }
}

/* Inter-layer expert affinity counts [MoE Inference Communication, §ExFlow 跨层专家
 * 亲和性]: for every token t, every expert i in its top-K at layer j and every expert p in its
 * top-K at layer j+1, cnt[i][p] += 1 (pre-drop routing decisions). The
 * conditional P(p | i) is cnt[i][p] / (number of tokens with i in their top-K
 * at layer j); each row of cnt sums to K times that number. */
EXPORT void orc_affinity(int64_t N, int64_t E, int64_t K, const int32_t *topk_j,
                         const int32_t *topk_j1, int64_t *cnt)
{
    for (int64_t t = 0; t < N; ++t)
        for (int64_t k = 0; k < K; ++k)
            for (int64_t q = 0; q < K; ++q)
                cnt[(int64_t)topk_j[t * K + k] * E + topk_j1[t * K + q]] += 1;
}

/* FP8 payload [MoE 推理服务工程真相 2026, §6.3 通信压缩: the token rows that cross the
 * all-to-all are sent as FP8 instead of BF16]. Format: e4m3 ("E4M3" of the OCP 8-bit floating-point formats):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 * subnormals m * 2^-9; no infinities; code 0x7F/0xFF is NaN, so 448 = 1.75 * 2^8 is the
 * largest finite value.
 *
 * Readings (the page names no scheme): one scale per row, a power of two, so that
 * dividing by it is exact; the scale is the smallest 2^j with amax(row) * 2^-j <= 448,
 * j clamped to [-126, 127] (a row of zeros, or a non-finite amax, takes j = 0); each
 * element is x * 2^-j rounded to the nearest e4m3 value, ties to the even code, values
 * beyond 448 saturated to 448. */

/* e4m3 value of a code. */
static double e4m3_value(uint8_t c)
{
    double s = (c & 0x80) ? -1.0 : 1.0;
    int ef = (c >> 3) & 15, m = c & 7;
    if (ef == 15 && m == 7)
        return NAN;
    if (ef == 0)
        return s * ldexp((double)m, -9);
    return s * ldexp(1.0 + m / 8.0, ef - 7);
}

/* Nearest e4m3 code to v (ties to even), saturating at +-448. */
static uint8_t e4m3_code(double v)
{
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    if (a > 448.0)
        return sign | 0x7E;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): the binade is [2^(e-1), 2^e) */
    int E = e - 1 < -6 ? -6 : e - 1;
    double quantum = ldexp(1.0, E - 3);       /* spacing of e4m3 values in this binade */
    double val = nearbyint(a / quantum) * quantum; /* exact quotient; ties to even */
    if (val > 448.0)
        val = 448.0;
    if (val == 0.0)
        return sign;
    frexp(val, &e);
    E = e - 1;
    if (E < -6)
        return sign | (uint8_t)(val / ldexp(1.0, -9)); /* subnormal: exponent field 0 */
    return sign | (uint8_t)((E + 7) << 3) | (uint8_t)(val / ldexp(1.0, E - 3) - 8.0);
}

EXPORT void orc_e4m3_encode(int64_t n, const double *v, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i)
        codes[i] = e4m3_code(v[i]);
}

EXPORT void orc_e4m3_decode(int64_t n, const uint8_t *codes, double *v)
{
    for (int64_t i = 0; i < n; ++i)
        v[i] = e4m3_value(codes[i]);
}

/* Scale exponent j of a row with largest magnitude amax. */
EXPORT int64_t orc_e4m3_scale_exponent(double amax)
{
    if (!(amax > 0.0) || !isfinite(amax))
        return 0;
    int64_t j = -126;
    while (j < 127 && ldexp(amax, (int)-j) > 448.0)
        j += 1;
    return j;
}

/* Row-wise quantisation of a bf16 matrix [rows][cols]: codes [rows][cols] and the
 * scale 2^j of each row (value = code value * scale). */
EXPORT void orc_quantize_rows_e4m3(int64_t rows, int64_t cols, const uint16_t *src,
                                   uint8_t *codes, float *scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double amax = 0.0;
        for (int64_t c = 0; c < cols; ++c) {
            double a = fabs((double)bf16_to_float(src[r * cols + c]));
            if (a > amax || isnan(a))
                amax = a;
        }
        int64_t j = orc_e4m3_scale_exponent(amax);
        scale[r] = (float)ldexp(1.0, (int)j);
        for (int64_t c = 0; c < cols; ++c)
            codes[r * cols + c] =
                e4m3_code(ldexp((double)bf16_to_float(src[r * cols + c]), (int)-j));
    }
}

/* Block-wise quantisation of the return payload [MoE 推理服务工程真相 2026, §6.3]: the rule of
 * orc_quantize_rows_e4m3 applied to every run of `block` consecutive columns of a row
 * instead of the whole row (reading: a row of expert outputs is produced in column tiles, a
 * block is not split across them). src [rows][cols] double; codes [rows][cols]; exps
 * [rows][cols / block] the exponent j of each block (value = code value * 2^j). */
EXPORT void orc_quantize_blocks_e4m3(int64_t rows, int64_t cols, int64_t block,
                                     const double *src, uint8_t *codes, int32_t *exps)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / block; ++b) {
            const double *v = src + r * cols + b * block;
            double amax = 0.0;
            for (int64_t c = 0; c < block; ++c) {
                double a = fabs(v[c]);
                if (a > amax || isnan(a))
                    amax = a;
            }
            int64_t j = orc_e4m3_scale_exponent(amax);
            exps[r * (cols / block) + b] = (int32_t)j;
            for (int64_t c = 0; c < block; ++c)
                codes[r * cols + b * block + c] = e4m3_code(ldexp(v[c], (int)-j));
        }
    }
}

/* Nearest fp16 value (1 sign, 5 exponent bits with bias 15, 10 mantissa bits: normal values
 * 2^-14 .. 65504, subnormals in steps of 2^-24) to a double, ties to even, as fp16 bits; a value
 * that rounds above 65504 becomes infinity. */
static uint16_t f16_nearest(double v)
{
    if (isnan(v))
        return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e); /* binade [2^(e-1), 2^e) */
    int E = e - 1 < -14 ? -14 : e - 1;
    double quantum = ldexp(1.0, E - 10);
    double val = nearbyint(a / quantum) * quantum; /* exact quotient; ties to even */
    if (val > 65504.0)
        return sign | 0x7C00;
    if (val == 0.0)
        return sign;
    frexp(val, &e);
    E = e - 1;
    if (E < -14) /* subnormal: exponent field 0, mantissa = val / 2^-24 */
        return sign | (uint16_t)(val / ldexp(1.0, -24));
    const uint16_t mant = (uint16_t)(ldexp(val, -E) * 1024.0 - 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

EXPORT void orc_round_f16(int64_t n, const double *v, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = f16_nearest(v[i]);
}

/* The exponent j of a block's power-of-two scale for fp16 codes: the smallest j in
 * [-126, 127] with amax * 2^-j <= 65504 (fp16's largest finite value), 0 for a zero or
 * non-finite amax: the e4m3 rule above with fp16's bound. */
EXPORT int64_t orc_f16_scale_exponent(double amax)
{
    if (!(amax > 0.0) || !isfinite(amax))
        return 0;
    int64_t j = -126;
    while (j < 127 && ldexp(amax, (int)-j) > 65504.0)
        j += 1;
    return j;
}

/* Block-wise fp16 quantisation of the expert outputs (the return payload in 16 bits, a reading
 * that extends the FP8 payload's block rule of [MoE 推理服务工程真相 2026, §6.3] to fp16 codes):
 * every run of `block` consecutive columns of a row takes the exponent j above from its largest
 * magnitude, each value is stored as the nearest fp16 of value * 2^-j. src [rows][cols] double;
 * codes [rows][cols] fp16 bits; exps [rows][cols / block] (value = code value * 2^j). */
EXPORT void orc_quantize_blocks_f16(int64_t rows, int64_t cols, int64_t block,
                                    const double *src, uint16_t *codes, int32_t *exps)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / block; ++b) {
            const double *v = src + r * cols + b * block;
            double amax = 0.0;
            for (int64_t c = 0; c < block; ++c) {
                double a = fabs(v[c]);
                if (a > amax || isnan(a))
                    amax = a;
            }
            int64_t j = orc_f16_scale_exponent(amax);
            exps[r * (cols / block) + b] = (int32_t)j;
            for (int64_t c = 0; c < block; ++c)
                codes[r * cols + b * block + c] = f16_nearest(ldexp(v[c], (int)-j));
        }
    }
}

/* Nearest bf16 value (1 sign, 8 exponent bits, 7 mantissa bits: binary32's range with 8
 * significant bits) to a double, ties to even, as bf16 bits; beyond the largest finite value
 * (2 - 2^-7) * 2^127 rounds to infinity. */
static uint16_t bf16_nearest(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e); /* binade [2^(e-1), 2^e) */
    int E = e - 1 < -126 ? -126 : e - 1;
    double quantum = ldexp(1.0, E - 7);
    double val = nearbyint(a / quantum) * quantum;
    if (val > ldexp(2.0 - ldexp(1.0, -7), 127))
        return sign | 0x7F80;
    float f = (float)val; /* exact: 8 significant bits within binary32's range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

EXPORT void orc_round_bf16(int64_t n, const double *v, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = bf16_nearest(v[i]);
}

/* Down projection alone, from bf16 activation rows: y[r][i] = sum_j h[r][j] * W2[e][i][j]
 * in fp64, e = row_expert[r]; W2 [E][d][f]. (The FP8 path's down projection runs on the
 * e4m3 rows of h, given here by their exact bf16 dequantisation.) */
EXPORT void orc_down_rows(int64_t nrows, const int32_t *row_expert, int64_t d, int64_t f,
                          const uint16_t *h, const uint16_t *w2, double *y_out)
{
#pragma omp parallel
    {
        double *hr = (double *)malloc((size_t)f * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t e = row_expert[r];
            for (int64_t j = 0; j < f; ++j)
                hr[j] = (double)bf16_to_float(h[r * f + j]);
            for (int64_t i = 0; i < d; ++i) {
                const uint16_t *c = w2 + (e * d + i) * f;
                double y = 0.0;
                for (int64_t j = 0; j < f; ++j)
                    y += hr[j] * (double)bf16_to_float(c[j]);
                y_out[r * d + i] = y;
            }
        }
        free(hr);
    }
}
