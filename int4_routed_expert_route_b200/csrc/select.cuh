// select.cuh -- noaux_tc group-limited top-k selection of one token by one
// warp ("Show HN: running GLM 5.2 on a slow computer", implemented features:
// DeepSeek-V3 style sigmoid router, noaux_tc, routed_scaling_factor).  Shared
// by the router kernels and the fused decode-layer kernel.
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

}  // namespace moe
