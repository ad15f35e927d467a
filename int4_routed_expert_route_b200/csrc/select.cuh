// select.cuh -- noaux_tc group-limited top-k selection ("Show HN: running GLM
// 5.2 on a slow computer", implemented features: DeepSeek-V3 style sigmoid
// router, noaux_tc, routed_scaling_factor), in two shapes that decide alike:
// one token by one warp (select_core, the router's large-batch kernel) and all
// tokens of a small batch by one block (select_tokens: the rank form at one
// token, the warp-reduction form from two on).  Shared by the router kernels
// and the fused decode-layer kernel.
#pragma once

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Selection: one warp per token.
// ---------------------------------------------------------------------------
struct SelArgs {
    const float *logits;  // [T][E] fp32
    int64_t T;
    const float *bias;
    int E, k, n_group, topk_group;
    float rsf, topp;
    int32_t *idx_out;
    float *w_out;
    float *gap_out;
};

// (value, index) argmax across the warp; ties go to the lower index.
static __device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

constexpr int SEL_WARPS = 4;

// Sigmoid score of one logit: evaluated in fp64, rounded to fp32.
static __device__ __forceinline__ float sigmoid_score(float logit) {
    return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(logit))));
}

// Selection of token t by one warp from its scores s_sm[E] and biased scores
// b_sm[E] in shared memory (read only); pick is 32 ints of scratch.
// Weights, optional top-p and the decision margin of token t from its picks
// (one thread): w = s[idx] / sum(s[picks]) * rsf in slot order.
// Weights of one token from its picks (one thread): w = s[idx] / sum(s[picks])
// * rsf with the sum in slot order; then the optional expert top-p: rank the
// slots by weight (ties keep slot order), keep the shortest prefix that reaches
// topp * total, drop the rest (index -1, weight 0), no renormalisation.
static __device__ void finish_weights(const float *s_sm, const int *pick, int k, float rsf, float topp,
                                      int32_t *idx, float *w) {
    float sum = 0.0f;
    for (int r = 0; r < k; r++)
        if (pick[r] >= 0) sum += s_sm[pick[r]];
    for (int r = 0; r < k; r++) {
        idx[r] = pick[r];
        w[r] = pick[r] >= 0 ? (s_sm[pick[r]] / sum) * rsf : 0.0f;
    }
    if (topp > 0.0f && topp < 1.0f) {
        float total = 0.0f;
        for (int r = 0; r < k; r++) total += w[r];
        const float target = topp * total;
        unsigned used = 0u, keep = 0u;
        float run = 0.0f;
        for (int r = 0; r < k; r++) {
            int best = -1;
            for (int j = 0; j < k; j++)
                if (!((used >> j) & 1u) && (best < 0 || w[j] > w[best])) best = j;
            used |= 1u << best;
            keep |= 1u << best;
            run += w[best];
            if (run >= target) break;
        }
        for (int r = 0; r < k; r++)
            if (!((keep >> r) & 1u)) {
                idx[r] = -1;
                w[r] = 0.0f;
            }
    }
}

static __device__ void select_finish(const SelArgs &a, int64_t t, const float *s_sm, const int *pick, float bk,
                              float rest, float last_kept, float best_dropped, bool any_dropped, int cand) {
    const int k = a.k;
    finish_weights(s_sm, pick, k, a.rsf, a.topp, a.idx_out + t * k, a.w_out + t * k);
    if (a.gap_out) {
        float gap = (cand > k) ? (bk - rest) : INFINITY;
        if (any_dropped) gap = fminf(gap, last_kept - best_dropped);
        a.gap_out[t] = gap;
    }
}

template <int MAXJ>  // candidate slots per lane: E <= 32 * MAXJ
static __device__ void select_core_j(const SelArgs &a, int64_t t, const float *s_sm, float *b_sm, int *pick) {
    const int lane = threadIdx.x & 31;
    const int E = a.E;

    const int ng = a.n_group, gsz = E / ng;
    float gscore = -INFINITY;
    if (lane < ng) {
        if (ng == 1) {
            gscore = 0.0f;
        } else {
            float t1 = -INFINITY, t2 = -INFINITY;
            for (int e = lane * gsz; e < (lane + 1) * gsz; e++) {
                const float b = b_sm[e];
                if (b > t1) {
                    t2 = t1;
                    t1 = b;
                } else if (b > t2) {
                    t2 = b;
                }
            }
            gscore = t1 + t2;
        }
    }
    // keep the topk_group best groups (ties to the lower group index)
    bool gsel = false;
    float last_kept = 0.0f;
    for (int r = 0; r < a.topk_group; r++) {
        float v = (lane < ng && !gsel) ? gscore : -INFINITY;
        int i = (lane < ng && !gsel) ? lane : 0x7fffffff;
        warp_argmax(v, i);
        if (lane == i) gsel = true;
        last_kept = v;
    }
    float best_dropped;
    {
        float v = (lane < ng && !gsel) ? gscore : -INFINITY;
        int i = lane;
        warp_argmax(v, i);
        best_dropped = v;
    }
    const bool any_dropped = ng > a.topk_group;
    const unsigned gmask = __ballot_sync(0xffffffffu, gsel);

    // top-k experts of b among the kept groups, descending, ties to lower index.
    // Each lane keeps its candidates e = lane + 32 j in registers with a
    // bitmask of the ones still selectable (kept group, not yet taken).
    const int nj = (E + 31) >> 5;
    float cb[MAXJ];
    uint32_t live = 0u;
#pragma unroll
    for (int j = 0; j < MAXJ; j++) {
        const int e = lane + 32 * j;
        cb[j] = -INFINITY;
        if (j < nj && e < E && ((gmask >> (e / gsz)) & 1u)) {
            cb[j] = b_sm[e];
            live |= 1u << j;
        }
    }
    float bk = 0.0f;
    for (int r = 0; r < a.k; r++) {
        float v = -INFINITY;
        int i = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < MAXJ; j++)
            if (((live >> j) & 1u) && (cb[j] > v || (cb[j] == v && lane + 32 * j < i))) {
                v = cb[j];
                i = lane + 32 * j;
            }
        warp_argmax(v, i);
        if (i >= E) i = -1;  // no candidate left (only with non-finite scores)
        if (lane == 0) pick[r] = i;
        if (i >= 0 && lane == (i & 31)) live &= ~(1u << (i >> 5));  // taken
        bk = v;
    }
    __syncwarp();
    float rest = -INFINITY;
    {
        int i = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < MAXJ; j++)
            if (((live >> j) & 1u) && (cb[j] > rest || (cb[j] == rest && lane + 32 * j < i))) {
                rest = cb[j];
                i = lane + 32 * j;
            }
        warp_argmax(rest, i);
    }
    const int cand = __popc(gmask) * gsz;
    if (lane == 0) select_finish(a, t, s_sm, pick, bk, rest, last_kept, best_dropped, any_dropped, cand);
}

static __device__ void select_core(const SelArgs &a, int64_t t, const float *s_sm, float *b_sm, int *pick) {
    if (a.E <= 256) select_core_j<8>(a, t, s_sm, b_sm, pick);
    else if (a.E <= 512) select_core_j<16>(a, t, s_sm, b_sm, pick);
    else select_core_j<32>(a, t, s_sm, b_sm, pick);
}

// Expert top-p of one token by its warp, the same decisions as finish_weights:
// lane r < k holds slot r's index and weight.  The total is summed in slot
// order and the running sum in rank order (descending weight, ties to the lower
// slot), each as one sequential fp32 chain that every lane repeats, so the
// roundings are finish_weights' own; the slot of rank i is kept when i = 0 or
// the sum of ranks below i is still short of topp * total.  Dropped slots get
// index -1 and weight 0.  A handful of shuffles instead of one lane's k^2 loop.
static __device__ __forceinline__ void topp_warp(int k, float topp, int lane, int &idx, float &w) {
    float total = 0.0f;
    for (int j = 0; j < k; j++) total += __shfl_sync(0xffffffffu, w, j);
    int rank = 0;
    for (int j = 0; j < k; j++) {
        const float o = __shfl_sync(0xffffffffu, w, j);
        rank += (o > w) || (o == w && j < lane);
    }
    float by_rank = 0.0f;  // lane i: the weight of rank i
    for (int j = 0; j < k; j++) {
        const float o = __shfl_sync(0xffffffffu, w, j);
        if (__shfl_sync(0xffffffffu, rank, j) == lane) by_rank = o;
    }
    const float target = topp * total;
    float run = 0.0f, before = 0.0f;
    for (int i = 0; i < k; i++) {
        if (lane == i) before = run;
        run += __shfl_sync(0xffffffffu, by_rank, i);
    }
    const bool keep_rank = lane == 0 || before < target;  // for rank = lane
    const bool keep = __shfl_sync(0xffffffffu, keep_rank ? 1 : 0, lane < k ? rank : 0) != 0;
    if (lane < k && !keep) {
        idx = -1;
        w = 0.0f;
    }
}

// Block-parallel group-limited top-k of T tokens from their scores s_all and
// biased scores b_all ([T][E] in shared memory), by nthr threads at once (a
// multiple of 32; Bar::sync() joins them): every (token, expert) finds its rank
// inside its group (the two best make the group score), every (token, group)
// its rank among the groups (the topk_group best are kept, ties to the lower
// group), and every candidate of a kept group its rank among the candidates
// (descending biased score, ties to the lower expert; four adjacent lanes split
// the comparisons): rank r < k is slot r.  Then the weights (finish_weights'
// arithmetic, one warp per token with the sum in slot order).  The same order
// and tie rules as select_core (top-p by topp_warp).  scratch holds T * (3 n_group + topk_group + k)
// words; idx_out / w_out [T][k] may be shared or global memory.
template <class Bar>
static __device__ __forceinline__ void select_block_ranks(const float *s_all, const float *b_all, int T, int E,
                                                          int k, int ng, int tkg, float rsf, float topp,
                                                          float *scratch, int32_t *idx_out, float *w_out, int tid,
                                                          int nthr) {
    const int gsz = E / ng, TE = T * E;
    float *gtop = scratch;                              // [T][ng][2]
    float *gsc = gtop + T * ng * 2;                     // [T][ng]
    int *kept = reinterpret_cast<int *>(gsc + T * ng);  // [T][tkg] kept groups
    int *pick = kept + T * tkg;                         // [T][k]
    for (int i = tid; i < T * k; i += nthr) pick[i] = -1;
    if (ng > 1) {
        for (int i = tid; i < TE; i += nthr) {
            const int t = i / E, e = i - t * E, g = e / gsz;
            const float *bt = b_all + t * E;
            const float be = bt[e];
            int rank = 0;
#pragma unroll 8
            for (int e2 = g * gsz; e2 < (g + 1) * gsz; e2++) {
                const float o = bt[e2];
                rank += (o > be) || (o == be && e2 < e);
            }
            if (rank < 2) gtop[(t * ng + g) * 2 + rank] = be;
        }
    }
    Bar::sync();
    for (int i = tid; i < T * ng; i += nthr) gsc[i] = ng == 1 ? 0.0f : gtop[2 * i] + gtop[2 * i + 1];
    Bar::sync();
    for (int i = tid; i < T * ng; i += nthr) {
        const int t = i / ng, g = i - t * ng;
        const float v = gsc[i];
        int rank = 0;
        for (int g2 = 0; g2 < ng; g2++) {
            const float o = gsc[t * ng + g2];
            rank += (o > v) || (o == v && g2 < g);
        }
        if (rank < tkg) kept[t * tkg + rank] = g;
    }
    Bar::sync();
    const int ncand = T * tkg * gsz;
    for (int base = tid & ~31; base < 4 * ncand; base += nthr) {  // warp-uniform trip count
        const int i0 = base + (tid & 31);
        const int i = i0 >> 2, part = i0 & 3;
        const bool live = i < ncand;
        int rank = 0, e = 0;
        if (live) {
            const int t = i / (tkg * gsz), rem = i - t * tkg * gsz;
            e = kept[t * tkg + rem / gsz] * gsz + rem % gsz;
            const float *bt = b_all + t * E;
            const float be = bt[e];
            for (int gi = part; gi < tkg; gi += 4) {  // part p compares with kept groups p, p + 4, ...
                const int e0 = kept[t * tkg + gi] * gsz;
#pragma unroll 8
                for (int e2 = e0; e2 < e0 + gsz; e2++) {
                    const float o = bt[e2];
                    rank += (o > be) || (o == be && e2 < e);
                }
            }
        }
        rank += __shfl_xor_sync(0xffffffffu, rank, 1);
        rank += __shfl_xor_sync(0xffffffffu, rank, 2);
        if (live && part == 0 && rank < k) pick[(i / (tkg * gsz)) * k + rank] = e;
    }
    Bar::sync();
    const int warp = tid >> 5, lane = tid & 31;
    for (int t = warp; t < T; t += nthr >> 5) {
        const int *pk = pick + t * k;
        const float *st = s_all + t * E;
        const int pr = lane < k ? pk[lane] : -1;
        const float sv = pr >= 0 ? st[pr] : 0.0f;
        float sum = 0.0f;
        for (int r = 0; r < k; r++) {
            const float o = __shfl_sync(0xffffffffu, sv, r);
            const int po = __shfl_sync(0xffffffffu, pr, r);
            if (po >= 0) sum += o;
        }
        int id = pr;
        float wv = pr >= 0 ? (sv / sum) * rsf : 0.0f;
        if (topp > 0.0f && topp < 1.0f) topp_warp(k, topp, lane, id, wv);
        if (lane < k) {
            idx_out[t * k + lane] = id;
            w_out[t * k + lane] = wv;
        }
    }
    Bar::sync();
}

struct BlockBar {
    static __device__ __forceinline__ void sync() { __syncthreads(); }
};

// Order-preserving 32-bit key of an fp32 value (a larger value has a larger
// unsigned key; -0 is folded into +0 so that the keys tie where the fp32
// comparison does), and its inverse.
static __device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
static __device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

constexpr int SELW_MAXC = 8;  // candidates per lane of select_block_warps

// select_block_warps applies when every group fits one warp's lanes, the group
// scores fit one warp and a token's candidates fit SELW_MAXC per lane.
static __host__ __device__ __forceinline__ bool select_warps_fit(int E, int k, int ng, int tkg) {
    const int gsz = E / ng, qpg = (gsz + 31) / 32;
    if (k > 32) return false;
    if (ng == 1) return qpg <= SELW_MAXC;
    return gsz <= 32 && ng <= 32 && tkg * qpg <= SELW_MAXC;
}

// Group-limited top-k of T tokens with warp reductions, the same result as
// select_block_ranks in two barrier phases:
//  1. one warp per (token, group): the group's two largest biased scores by two
//     unsigned max-reductions over order keys (the second is the first again
//     when two lanes hold it); lane 0 stores their fp32 sum;
//  2. one warp per token: lane g ranks group g among the group scores (ties to
//     the lower group) and a ballot gives the kept groups; every lane then holds
//     the candidates j = lane, lane + 32, ... of each kept group (ascending
//     expert order), and k rounds take the largest key (max-reduction) and,
//     among the lanes holding it, the lowest expert (min-reduction): round r
//     gives slot r.  Then the weights as in select_block_ranks.
// Its rounds are serial, so it pays off where several tokens run side by side.
// scratch: T * (n_group + k) words.
template <class Bar>
static __device__ __forceinline__ void select_block_warps(const float *s_all, const float *b_all, int T, int E,
                                                          int k, int ng, int tkg, float rsf, float topp,
                                                          float *scratch, int32_t *idx_out, float *w_out, int tid,
                                                          int nthr) {
    const int gsz = E / ng;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
    constexpr int NONE = 0x7fffffff;
    float *gsc = scratch;                               // [T][ng]
    int *pick = reinterpret_cast<int *>(gsc + T * ng);  // [T][k]
    if (ng > 1) {
        for (int task = warp; task < T * ng; task += nwarps) {
            const int t = task / ng, g = task - t * ng;
            const uint32_t key = lane < gsz ? order_key(b_all[t * E + g * gsz + lane]) : 0u;
            const uint32_t m1 = __reduce_max_sync(0xffffffffu, key);
            const uint32_t hold = __ballot_sync(0xffffffffu, key == m1);
            const uint32_t m2 = __popc(hold) >= 2 ? m1 : __reduce_max_sync(0xffffffffu, key == m1 ? 0u : key);
            if (lane == 0) gsc[task] = key_value(m1) + key_value(m2);
        }
        Bar::sync();
    }
    for (int t = warp; t < T; t += nwarps) {
        const float *bt = b_all + t * E;
        uint32_t kept = 1u;
        if (ng > 1) {
            const float v = lane < ng ? gsc[t * ng + lane] : 0.0f;
            int rank = 0;
            for (int g2 = 0; g2 < ng; g2++) {
                const float o = __shfl_sync(0xffffffffu, v, g2);
                rank += (o > v) || (o == v && g2 < lane);
            }
            kept = __ballot_sync(0xffffffffu, lane < ng && rank < tkg);
        }
        // slot c of a lane: kept group number c / qpg (ascending), j = lane + 32 (c % qpg)
        const int qpg = (gsz + 31) >> 5;
        uint32_t ck[SELW_MAXC], avail = 0u, km = kept;
        int ce[SELW_MAXC], g = -1, q = qpg;
#pragma unroll
        for (int c = 0; c < SELW_MAXC; c++) {
            if (q == qpg) {
                q = 0;
                g = km ? __ffs(km) - 1 : -1;
                km &= km - 1;
            }
            const int j = lane + 32 * q;
            const bool ok = g >= 0 && j < gsz;
            ck[c] = ok ? order_key(bt[g * gsz + j]) : 0u;
            ce[c] = ok ? g * gsz + j : NONE;
            avail |= static_cast<uint32_t>(ok) << c;
            q++;
        }
        int mine = -1;
        for (int r = 0; r < k; r++) {
            uint32_t bk = 0u;
            int be = NONE;
#pragma unroll
            for (int c = 0; c < SELW_MAXC; c++)
                if (((avail >> c) & 1u) && (ck[c] > bk || (ck[c] == bk && ce[c] < be))) {
                    bk = ck[c];
                    be = ce[c];
                }
            const uint32_t top = __reduce_max_sync(0xffffffffu, bk);
            const int win = static_cast<int>(
                __reduce_min_sync(0xffffffffu, bk == top ? static_cast<uint32_t>(be) : static_cast<uint32_t>(NONE)));
#pragma unroll
            for (int c = 0; c < SELW_MAXC; c++)
                if (ce[c] == win) avail &= ~(1u << c);
            if (lane == r) mine = win == NONE ? -1 : win;
        }
        if (lane < k) pick[t * k + lane] = mine;
        const float *st = s_all + t * E;
        const float sv = mine >= 0 ? st[mine] : 0.0f;
        float sum = 0.0f;
        for (int r = 0; r < k; r++) {
            const float o = __shfl_sync(0xffffffffu, sv, r);
            if (__shfl_sync(0xffffffffu, mine, r) >= 0) sum += o;
        }
        int id = mine;
        float wv = mine >= 0 ? (sv / sum) * rsf : 0.0f;
        if (topp > 0.0f && topp < 1.0f) topp_warp(k, topp, lane, id, wv);
        if (lane < k) {
            idx_out[t * k + lane] = id;
            w_out[t * k + lane] = wv;
        }
    }
    Bar::sync();
}

// Words of selection scratch per token (either form of select_tokens).
static __host__ __device__ __forceinline__ int select_scratch_words(int E, int k, int ng, int tkg) {
    (void)E;
    return 3 * ng + tkg + k;
}

// Group-limited top-k of T tokens by nthr threads (Bar::sync() joins them):
// from two tokens on the warp-reduction form where the configuration fits it
// and has at most 16 groups (1.3 times faster than the rank form at two tokens
// of 256 experts in 8 groups, three times at eight), else the rank form (the
// faster of the two for one token, and with many small groups).
// scratch: T * select_scratch_words() words.
template <class Bar>
static __device__ __forceinline__ void select_tokens(const float *s_all, const float *b_all, int T, int E, int k,
                                                     int ng, int tkg, float rsf, float topp, float *scratch,
                                                     int32_t *idx_out, float *w_out, int tid, int nthr) {
    if (T >= 2 && ng <= 16 && select_warps_fit(E, k, ng, tkg))
        select_block_warps<Bar>(s_all, b_all, T, E, k, ng, tkg, rsf, topp, scratch, idx_out, w_out, tid, nthr);
    else
        select_block_ranks<Bar>(s_all, b_all, T, E, k, ng, tkg, rsf, topp, scratch, idx_out, w_out, tid, nthr);
}

}  // namespace moe
