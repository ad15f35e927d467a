/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for the routed-expert
 * MoE layer (sigmoid noaux_tc router, int4/int8/int2 per-row quantised SwiGLU
 * experts, shared expert, batch-union bucketing).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file;
 * only the tests, the package smoke check and the CPU-baseline leg of the
 * benchmark load it.  It shares no code, header or table with the CUDA library.
 *
 * Sources (the pages describe the method; none prints code for it):
 *  - "Show HN: running GLM 5.2 on a slow computer" (hi.news.hada.io), section
 *    "implemented features": DeepSeek-V3 style sigmoid router with noaux_tc,
 *    routed_scaling_factor and a shared expert; int8/int4/int2 quantisation with
 *    per-row scales, dequant-on-use; batch-union MoE (each unique expert of a
 *    batch is read once and applied to every position routed to it).
 *  - "Enthusiast ran GLM-5.2 on a laptop with 25 GB of RAM" (ideipro.ru):
 *    8 experts per token per MoE layer; int8/int4/int2 kernels with per-row
 *    scales whose packing is checked bit for bit.
 *  - The workload statement of this layer fixes the int4 scheme (scale =
 *    max|row|/7, q = clamp(round(w/scale), -8, 7), stored as q+8 with the low
 *    nibble holding the even column), the int2 scheme (q in [-2,1], scale =
 *    max|row|/1.5) and the SwiGLU form y = W_down(silu(W_gate x) * W_up x).
 *
 * Precision: every floating-point step is fp64, except the steps that decide an
 * integer (a quantised code, a routing choice).  Those are taken in fp32, the
 * precision the kernels decide in:
 *  - quantisation: s = m / Qmax and q = roundf(w / s), fp32 IEEE divisions;
 *  - routing: logit = fp32(exact dot product), s = fp32(sigmoid(logit) in fp64),
 *    b = s + bias in fp32, group score = top1 + top2 in fp32, comparisons in fp32,
 *    weights w_i = (s_i / sum_i s_i) * rsf in fp32 with the sum in slot order.
 * Readings where the pages are silent are listed in the design notes and in the
 * comments below.
 *
 * The expert top-p step (route_one) follows a reading of an option the pages
 * name ("--topp 0.7") without defining it: rank the slots by weight, keep the
 * shortest prefix reaching topp * total, drop the rest without renormalising.
 * That reading is pinned by properties checked on random weight vectors (the
 * kept slots are a prefix of the weight order, their sum reaches the target, a
 * prefix one slot shorter does not, kept weights are unchanged, dropped slots
 * read -1 / 0) and by hand-worked golden cases; the rule itself stays a reading.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_EMISSING 2

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the expert FFN rows are split over (1 = serial).  Every output value
 * is computed by one thread in the order written here, whatever the count. */
void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ */
/* bf16 helpers                                                        */
/* ------------------------------------------------------------------ */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* The bf16 value nearest to the double v, ties to the even mantissa.  The two
 * bf16 candidates are found from the fp32 rounding of v; the choice between them
 * is made on v itself, so no double rounding can occur. */
uint16_t orc_double_to_bf16(double v)
{
    float f = (float)v; /* fp32 has 24 bits; a bf16 tie is decided below on the double */
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) /* inf / nan */
        return (uint16_t)(u >> 16);
    /* candidates: truncation and next bf16 up (in magnitude) */
    uint32_t lo = u & 0xffff0000u;
    uint32_t hi = lo + 0x00010000u;
    float flo, fhi;
    memcpy(&flo, &lo, 4);
    memcpy(&fhi, &hi, 4);
    double dlo = fabs(v - (double)flo), dhi = fabs(v - (double)fhi);
    if (dlo < dhi) return (uint16_t)(lo >> 16);
    if (dhi < dlo) return (uint16_t)(hi >> 16);
    return (uint16_t)(((lo >> 16) & 1u) ? (hi >> 16) : (lo >> 16));
}

/* ------------------------------------------------------------------ */
/* Quantisation, packing, dequantisation                               */
/* ------------------------------------------------------------------ */

static int qrange(int bits, float *qmax_div, int *qlo, int *qhi)
{
    switch (bits) {
    case 4: *qmax_div = 7.0f;   *qlo = -8;   *qhi = 7;   return 0;
    case 8: *qmax_div = 127.0f; *qlo = -128; *qhi = 127; return 0;
    case 2: *qmax_div = 1.5f;   *qlo = -2;   *qhi = 1;   return 0;
    default: return -1;
    }
}

int64_t orc_row_bytes(int bits, int64_t cols)
{
    return (cols * bits + 7) / 8;
}

/* Store code q (already in range) of column j into a packed row.
 * int4: byte j/2 holds column 2m in its low nibble and 2m+1 in its high nibble,
 *       each as q+8 (the stated storage rule).
 * int2: byte j/4 holds columns 4m..4m+3 in bit pairs 0-1, 2-3, 4-5, 6-7 (lowest
 *       bits = lowest column, by analogy with int4), each as q+2.
 * int8: one two's-complement byte per column. */
static void put_code(uint8_t *row, int bits, int64_t j, int q)
{
    if (bits == 8) {
        row[j] = (uint8_t)(int8_t)q;
    } else if (bits == 4) {
        uint8_t v = (uint8_t)(q + 8);
        if (j % 2 == 0) row[j / 2] = (uint8_t)((row[j / 2] & 0xf0u) | v);
        else            row[j / 2] = (uint8_t)((row[j / 2] & 0x0fu) | (v << 4));
    } else { /* 2 */
        uint8_t v = (uint8_t)(q + 2);
        int sh = (int)(j % 4) * 2;
        row[j / 4] = (uint8_t)((row[j / 4] & ~(3u << sh)) | (v << sh));
    }
}

static int get_code(const uint8_t *row, int bits, int64_t j)
{
    if (bits == 8) return (int)(int8_t)row[j];
    if (bits == 4) {
        uint8_t b = row[j / 2];
        return (int)((j % 2 == 0) ? (b & 0x0f) : (b >> 4)) - 8;
    }
    uint8_t b = row[j / 4];
    return (int)((b >> ((j % 4) * 2)) & 3u) - 2;
}

int orc_pack(const int32_t *q, int64_t rows, int64_t cols, int bits, uint8_t *out)
{
    float d; int lo, hi;
    if (qrange(bits, &d, &lo, &hi)) return ORC_EINVAL;
    if (cols % (8 / bits) != 0 && bits != 8) return ORC_EINVAL;
    int64_t rb = orc_row_bytes(bits, cols);
    memset(out, 0, (size_t)(rb * rows));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols; j++) {
            int v = q[r * cols + j];
            if (v < lo || v > hi) return ORC_EINVAL;
            put_code(out + r * rb, bits, j, v);
        }
    return ORC_OK;
}

int orc_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int bits, int32_t *q)
{
    float d; int lo, hi;
    if (qrange(bits, &d, &lo, &hi)) return ORC_EINVAL;
    if (cols % (8 / bits) != 0 && bits != 8) return ORC_EINVAL;
    int64_t rb = orc_row_bytes(bits, cols);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols; j++)
            q[r * cols + j] = get_code(packed + r * rb, bits, j);
    return ORC_OK;
}

/* Per-row symmetric quantisation (stated scheme; rounding reading below).
 *   m = max_j |w_j|                   (fp32, exact)
 *   m == 0  ->  s = 0 and every q = 0  (reading: the formula divides by zero)
 *   s = m / Qmax                       (fp32 IEEE division)
 *   q_j = clamp(roundf(w_j / s), qlo, qhi)
 * roundf rounds halves away from zero (reading: the engine is plain C and
 * rounds with the C library; the pages name no other rule). */
int orc_quantize_rows(const float *w, int64_t rows, int64_t cols, int bits,
                      uint8_t *q_out, float *scale_out)
{
    float qmax_div; int lo, hi;
    if (qrange(bits, &qmax_div, &lo, &hi)) return ORC_EINVAL;
    if (bits == 4 && cols % 2) return ORC_EINVAL;
    if (bits == 2 && cols % 4) return ORC_EINVAL;
    int64_t rb = orc_row_bytes(bits, cols);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        const float *wr = w + r * cols;
        uint8_t *qr = q_out + r * rb;
        float m = 0.0f;
        for (int64_t j = 0; j < cols; j++) {
            float a = fabsf(wr[j]);
            if (a > m) m = a;
        }
        float s = (m == 0.0f) ? 0.0f : m / qmax_div;
        scale_out[r] = s;
        memset(qr, 0, (size_t)rb);
        for (int64_t j = 0; j < cols; j++) {
            int q = 0;
            if (s != 0.0f) {
                float v = wr[j] / s;
                float rv = roundf(v);
                q = (int)rv;
                if (q < lo) q = lo;
                if (q > hi) q = hi;
            }
            put_code(qr, bits, j, q);
        }
    }
    return ORC_OK;
}

/* Dequantised weight as the exact product q * s (fp64 holds it exactly). */
static double deq(const uint8_t *row, const float *scale, int64_t r, int bits, int64_t j)
{
    return (double)get_code(row, bits, j) * (double)scale[r];
}

int orc_dequant_rows(const uint8_t *packed, const float *scale, int64_t rows, int64_t cols,
                     int bits, double *out)
{
    float d; int lo, hi;
    if (qrange(bits, &d, &lo, &hi)) return ORC_EINVAL;
    int64_t rb = orc_row_bytes(bits, cols);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < cols; j++)
            out[r * cols + j] = deq(packed + r * rb, scale, r, bits, j);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Router: sigmoid scores, noaux_tc bias-corrected group-limited top-k  */
/* ------------------------------------------------------------------ */

/* Scores of one token.
 *   logit_e = sum_j G[e,j] * x_j    exact products, fp64 sum, rounded to fp32
 *   s_e     = sigmoid(logit_e)      evaluated in fp64, rounded to fp32
 * (reading: the pages fix no router precision; the decision is taken on fp32
 *  scores and the scores themselves are the fp32 roundings of the exact values.) */
static void token_scores(const uint16_t *x, int64_t H, const float *G, int E, float *s)
{
    for (int e = 0; e < E; e++) {
        double acc = 0.0;
        for (int64_t j = 0; j < H; j++)
            acc += (double)G[(int64_t)e * H + j] * bf16_to_double(x[j]);
        float logit = (float)acc;
        s[e] = (float)(1.0 / (1.0 + exp(-(double)logit)));
    }
}

/* Route one token given its fp32 sigmoid scores s[E].
 *  b_e = s_e + bias_e (fp32); the bias only steers the choice (noaux_tc).
 *  Groups are the n_group contiguous blocks of E/n_group experts (reading).
 *  Group score = (largest b in the group) + (second largest b), fp32.
 *  The topk_group best groups are kept, ties to the lower group index (reading).
 *  Experts outside the kept groups are not candidates (reading).
 *  idx = the k candidates of largest b, in descending b, ties to the lower
 *  expert index (reading: the order must be fixed to compare indices exactly).
 *  w_i = (s_{idx_i} / sum_i s_{idx_i}) * rsf, unbiased scores, fp32, sum in slot
 *  order (reading: normalisation is implied by the weights summing to rsf).
 *  gap  = b_(k) - max b of the candidates not chosen   (INFINITY if none)
 *  ggap = score of the last kept group - best score of a dropped group (INF if none)
 *  Expert top-p (topp in (0,1)): the slots are ranked by w descending (ties to
 *  the lower slot); the shortest prefix whose weight sum reaches topp * sum(w)
 *  is kept; the other slots get idx = -1 and w = 0; no renormalisation
 *  (reading of the "--topp" option: the pages do not define it). */
static int route_one(const float *s, const float *bias, int E, int k, int n_group, int topk_group,
                     float rsf, float topp, int32_t *idx, float *w, double *gap, double *ggap,
                     int32_t *group_sel)
{
    float b[4096];
    float gscore[1024];
    int gsel[1024];
    int chosen[4096];
    if (E > 4096 || n_group > 1024) return ORC_EINVAL;
    int gs = E / n_group;
    for (int e = 0; e < E; e++) b[e] = s[e] + bias[e];

    for (int g = 0; g < n_group; g++) {
        float t1 = -INFINITY, t2 = -INFINITY;
        for (int e = g * gs; e < (g + 1) * gs; e++) {
            if (b[e] > t1) { t2 = t1; t1 = b[e]; }
            else if (b[e] > t2) { t2 = b[e]; }
        }
        gscore[g] = (n_group == 1) ? 0.0f : (t1 + t2);
        gsel[g] = 0;
    }
    int last_group = -1;
    for (int r = 0; r < topk_group; r++) {
        int best = -1;
        for (int g = 0; g < n_group; g++) {
            if (gsel[g]) continue;
            if (best < 0 || gscore[g] > gscore[best]) best = g;
        }
        gsel[best] = 1;
        last_group = best;
    }
    {
        double bestrest = -INFINITY;
        int any = 0;
        for (int g = 0; g < n_group; g++)
            if (!gsel[g]) { any = 1; if ((double)gscore[g] > bestrest) bestrest = gscore[g]; }
        *ggap = any ? (double)gscore[last_group] - bestrest : INFINITY;
    }
    if (group_sel)
        for (int g = 0; g < n_group; g++) group_sel[g] = gsel[g];

    for (int e = 0; e < E; e++) chosen[e] = 0;
    for (int i = 0; i < k; i++) {
        int best = -1;
        for (int e = 0; e < E; e++) {
            if (chosen[e] || !gsel[e / gs]) continue;
            if (best < 0 || b[e] > b[best]) best = e;
        }
        if (best < 0) return ORC_EINVAL;
        chosen[best] = 1;
        idx[i] = best;
    }
    {
        double bestrest = -INFINITY;
        int any = 0;
        for (int e = 0; e < E; e++)
            if (!chosen[e] && gsel[e / gs]) { any = 1; if ((double)b[e] > bestrest) bestrest = b[e]; }
        *gap = any ? (double)b[idx[k - 1]] - bestrest : INFINITY;
    }

    float sum = 0.0f;
    for (int i = 0; i < k; i++) sum += s[idx[i]];
    for (int i = 0; i < k; i++) w[i] = (s[idx[i]] / sum) * rsf;

    if (topp > 0.0f && topp < 1.0f) {
        int order[4096], keep[4096], used[4096];
        float total = 0.0f;
        for (int i = 0; i < k; i++) { keep[i] = 0; used[i] = 0; }
        /* rank slots by w descending; a strict comparison keeps ties in slot order */
        for (int i = 0; i < k; i++) {
            int best = -1;
            for (int j = 0; j < k; j++)
                if (!used[j] && (best < 0 || w[j] > w[best])) best = j;
            used[best] = 1;
            order[i] = best;
        }
        for (int i = 0; i < k; i++) total += w[i];
        float target = topp * total;
        float run = 0.0f;
        for (int i = 0; i < k; i++) {
            keep[order[i]] = 1;
            run += w[order[i]];
            if (run >= target) break;
        }
        for (int i = 0; i < k; i++)
            if (!keep[i]) { idx[i] = -1; w[i] = 0.0f; }
    }
    return ORC_OK;
}

static int check_router_cfg(int E, int k, int n_group, int topk_group)
{
    if (E < 1 || E > 4096 || k < 1 || n_group < 1 || topk_group < 1) return ORC_EINVAL;
    if (E % n_group) return ORC_EINVAL;
    if (topk_group > n_group) return ORC_EINVAL;
    if (n_group > 1 && E / n_group < 2) return ORC_EINVAL;
    if (k > topk_group * (E / n_group)) return ORC_EINVAL;
    return ORC_OK;
}

/* Full router over T tokens.  scores_out [T,E] (nullable) receives the fp32
 * sigmoid scores; gap/ggap [T] (nullable) the decision margins. */
int orc_route(const uint16_t *x, int64_t T, int64_t H, const float *G, const float *bias,
              int E, int k, int n_group, int topk_group, float rsf, float topp,
              int32_t *idx_out, float *w_out, double *gap_out, double *ggap_out,
              float *scores_out)
{
    if (check_router_cfg(E, k, n_group, topk_group)) return ORC_EINVAL;
    int err = 0;
    for (int64_t t = 0; t < T; t++) {
        float *s = (float *)malloc(sizeof(float) * (size_t)E);
        double gap, ggap;
        token_scores(x + t * H, H, G, E, s);
        if (scores_out) memcpy(scores_out + t * E, s, sizeof(float) * (size_t)E);
        if (route_one(s, bias, E, k, n_group, topk_group, rsf, topp,
                      idx_out + t * k, w_out + t * k, &gap, &ggap, NULL))
            err = 1;
        if (gap_out) gap_out[t] = gap;
        if (ggap_out) ggap_out[t] = ggap;
        free(s);
    }
    return err ? ORC_EINVAL : ORC_OK;
}

/* Router decision from given fp32 scores (used by the brute-force pins). */
int orc_route_from_scores(const float *s, int64_t T, const float *bias, int E, int k, int n_group,
                          int topk_group, float rsf, float topp, int32_t *idx_out, float *w_out,
                          double *gap_out, double *ggap_out, int32_t *group_sel_out)
{
    if (check_router_cfg(E, k, n_group, topk_group)) return ORC_EINVAL;
    for (int64_t t = 0; t < T; t++) {
        double gap, ggap;
        if (route_one(s + t * E, bias, E, k, n_group, topk_group, rsf, topp, idx_out + t * k,
                      w_out + t * k, &gap, &ggap,
                      group_sel_out ? group_sel_out + t * n_group : NULL))
            return ORC_EINVAL;
        if (gap_out) gap_out[t] = gap;
        if (ggap_out) ggap_out[t] = ggap;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Batch-union bucketing: a stable counting sort of (token, slot) pairs */
/* ------------------------------------------------------------------ */

/* pair p = t*k + slot.  list = all p, grouped by expert ascending and, inside an
 * expert, in increasing p (hence increasing token).  offsets[e]..offsets[e+1]
 * delimit expert e.  unique = experts with at least one pair, ascending.
 * Pairs with idx < 0 (dropped by expert top-p) are not listed. */
int orc_bucket(const int32_t *idx, int64_t T, int k, int E, int32_t *counts, int32_t *offsets,
               int32_t *list, int32_t *unique, int32_t *n_unique)
{
    int64_t P = T * k;
    for (int64_t p = 0; p < P; p++)
        if (idx[p] >= E) return ORC_EINVAL;
    int64_t pos = 0;
    int nu = 0;
    for (int e = 0; e < E; e++) {
        offsets[e] = (int32_t)pos;
        int c = 0;
        for (int64_t p = 0; p < P; p++)
            if (idx[p] == e) { list[pos++] = (int32_t)p; c++; }
        counts[e] = c;
        if (c > 0) unique[nu++] = e;
    }
    offsets[E] = (int32_t)pos;
    *n_unique = nu;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* SwiGLU expert FFN and the MoE layer                                  */
/* ------------------------------------------------------------------ */

typedef struct {
    const uint8_t *qg; const float *sg;
    const uint8_t *qu; const float *su;
    const uint8_t *qd; const float *sd;
    int bits;
} orc_expert;

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* y[H] = W'_d ( silu(W'_g x) * (W'_u x) ), W' = q*s exactly, all fp64.
 * Gate/up are [I,H], down is [H,I], row-major packed. */
static void ffn_token(const orc_expert *ex, const double *x, int64_t H, int64_t I, double *h,
                      double *y)
{
    int64_t rbh = orc_row_bytes(ex->bits, H), rbi = orc_row_bytes(ex->bits, I);
    /* rows are independent: each is computed by one thread */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        const uint8_t *rg = ex->qg + i * rbh, *ru = ex->qu + i * rbh;
        for (int64_t j = 0; j < H; j++) {
            g += deq(rg, ex->sg, i, ex->bits, j) * x[j];
            u += deq(ru, ex->su, i, ex->bits, j) * x[j];
        }
        h[i] = silu(g) * u;
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < H; j++) {
        double acc = 0.0;
        const uint8_t *rd = ex->qd + j * rbi;
        for (int64_t i = 0; i < I; i++) acc += deq(rd, ex->sd, j, ex->bits, i) * h[i];
        y[j] = acc;
    }
}

int orc_expert_ffn(const uint16_t *x, int64_t T, int64_t H, int64_t I, const uint8_t *qg,
                   const float *sg, const uint8_t *qu, const float *su, const uint8_t *qd,
                   const float *sd, int bits, double *y_out)
{
    orc_expert ex = {qg, sg, qu, su, qd, sd, bits};
    float d; int lo, hi;
    if (qrange(bits, &d, &lo, &hi)) return ORC_EINVAL;
    for (int64_t t = 0; t < T; t++) {
        double *xd = (double *)malloc(sizeof(double) * (size_t)H);
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        for (int64_t j = 0; j < H; j++) xd[j] = bf16_to_double(x[t * H + j]);
        ffn_token(&ex, xd, H, I, h, y_out + t * H);
        free(xd);
        free(h);
    }
    return ORC_OK;
}

/* MoE layer: y_t = sum_i w_{t,i} FFN_{idx_{t,i}}(x_t) + FFN_shared(x_t).
 * The shared expert is added unweighted (reading of "shared expert").
 * Routing comes from orc_route unless idx_in/w_in are given (teacher forcing).
 * Experts are given as arrays of E pointers; an expert may be NULL when no token
 * selects it (the call fails with ORC_EMISSING otherwise). */
int orc_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, const float *G,
              const float *bias, int E, int k, int n_group, int topk_group, float rsf, float topp,
              const uint8_t *const *qg, const float *const *sg, const uint8_t *const *qu,
              const float *const *su, const uint8_t *const *qd, const float *const *sd, int bits,
              const uint8_t *sh_qg, const float *sh_sg, const uint8_t *sh_qu, const float *sh_su,
              const uint8_t *sh_qd, const float *sh_sd, int sh_bits,
              const int32_t *idx_in, const float *w_in, double *y_out, int32_t *idx_out,
              float *w_out)
{
    int rc;
    if (idx_in) {
        memcpy(idx_out, idx_in, sizeof(int32_t) * (size_t)(T * k));
        memcpy(w_out, w_in, sizeof(float) * (size_t)(T * k));
    } else {
        rc = orc_route(x, T, H, G, bias, E, k, n_group, topk_group, rsf, topp, idx_out, w_out,
                       NULL, NULL, NULL);
        if (rc) return rc;
    }
    for (int64_t p = 0; p < T * k; p++) {
        int e = idx_out[p];
        if (e >= E) return ORC_EINVAL;
        if (e >= 0 && (!qg[e] || !sg[e] || !qu[e] || !su[e] || !qd[e] || !sd[e])) return ORC_EMISSING;
    }
    int err = 0;
    for (int64_t t = 0; t < T; t++) {
        double *xd = (double *)malloc(sizeof(double) * (size_t)H);
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *ye = (double *)malloc(sizeof(double) * (size_t)H);
        double *yt = y_out + t * H;
        for (int64_t j = 0; j < H; j++) { xd[j] = bf16_to_double(x[t * H + j]); yt[j] = 0.0; }
        for (int i = 0; i < k; i++) {
            int e = idx_out[t * k + i];
            if (e < 0) continue;
            orc_expert ex = {qg[e], sg[e], qu[e], su[e], qd[e], sd[e], bits};
            ffn_token(&ex, xd, H, I, h, ye);
            double wi = (double)w_out[t * k + i];
            for (int64_t j = 0; j < H; j++) yt[j] += wi * ye[j];
        }
        if (sh_qg) {
            orc_expert ex = {sh_qg, sh_sg, sh_qu, sh_su, sh_qd, sh_sd, sh_bits};
            ffn_token(&ex, xd, H, I, h, ye);
            for (int64_t j = 0; j < H; j++) yt[j] += ye[j];
        }
        free(xd);
        free(h);
        free(ye);
    }
    return err ? ORC_EINVAL : ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Stack pieces: RMSNorm (gamma = 1) and the bf16 layer input            */
/* ------------------------------------------------------------------ */

/* out_t = v_t / sqrt(mean_j v_tj^2 + eps), fp64; then rounded to bf16, the
 * dtype the layer takes (reading: the pages give no norm weight, so gamma = 1). */
int orc_rmsnorm_bf16(const double *v, int64_t T, int64_t H, double eps, uint16_t *out,
                     double *out_f64)
{
    for (int64_t t = 0; t < T; t++) {
        double ss = 0.0;
        for (int64_t j = 0; j < H; j++) ss += v[t * H + j] * v[t * H + j];
        double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t j = 0; j < H; j++) {
            double o = v[t * H + j] * r;
            if (out_f64) out_f64[t * H + j] = o;
            if (out) out[t * H + j] = orc_double_to_bf16(o);
        }
    }
    return ORC_OK;
}
