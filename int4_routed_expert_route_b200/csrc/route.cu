// route.cu -- sigmoid router with noaux_tc bias-corrected group-limited top-k.
//
// "Show HN: running GLM 5.2 on a slow computer", implemented features: a
// DeepSeek-V3 style sigmoid router (noaux_tc, routed_scaling_factor, shared
// expert).  Per token: logits G.x, s = sigmoid(logit), b = s + bias chooses the
// experts (groups ranked by the sum of their two best b, topk_group groups
// kept, top-k experts of b inside them), weights are the unbiased s of the
// chosen experts normalised to routed_scaling_factor.
//
// Precision: a logit is the exact dot product rounded to fp32 (fp64
// accumulation of exact bf16*fp32 products for small batches; for large
// batches fp32 chains of 32 products folded into fp64, error < ~1e-6 of the
// fp32 ulp budget the near-tie flag allows), the sigmoid is evaluated in fp64
// and rounded to fp32, every decision compares fp32 values.  No fast-math.
#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits for small batches: one warp per (expert, K-slice); the warp keeps its
// slice of the gate row in registers and loops over the tokens.
// part[ks][t][e] = sum over the slice of G[e,j] * x[t,j], fp64.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) route_logits_small(const uint16_t *__restrict__ x,
                                                          int64_t T, int64_t H,
                                                          const float *__restrict__ G, int E,
                                                          int KS, double *__restrict__ part) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int ks = blockIdx.y;
    if (e >= E) return;
    const int64_t L = H / KS;
    const int64_t k0 = static_cast<int64_t>(ks) * L;
    constexpr int MAXV = 4;  // up to 4 float4 per lane held in registers (L <= 512)
    float4 g[MAXV];
    int nv = 0;
#pragma unroll
    for (int v = 0; v < MAXV; v++) {
        const int64_t j = 4 * lane + 128 * v;
        if (j < L) {
            g[v] = *reinterpret_cast<const float4 *>(G + static_cast<int64_t>(e) * H + k0 + j);
            nv = v + 1;
        } else {
            g[v] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    for (int64_t t = 0; t < T; t++) {
        double acc = 0.0;
        const uint16_t *xr = x + t * H + k0;
#pragma unroll
        for (int v = 0; v < MAXV; v++) {
            if (v < nv) {
                const int64_t j = 4 * lane + 128 * v;
                if (j < L) {
                    const uint2 xv = *reinterpret_cast<const uint2 *>(xr + j);
                    acc = fma(static_cast<double>(g[v].x), static_cast<double>(bf16_bits_to_float(xv.x & 0xffffu)), acc);
                    acc = fma(static_cast<double>(g[v].y), static_cast<double>(bf16_bits_to_float(xv.x >> 16)), acc);
                    acc = fma(static_cast<double>(g[v].z), static_cast<double>(bf16_bits_to_float(xv.y & 0xffffu)), acc);
                    acc = fma(static_cast<double>(g[v].w), static_cast<double>(bf16_bits_to_float(xv.y >> 16)), acc);
                }
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) part[(static_cast<int64_t>(ks) * T + t) * E + e] = acc;
    }
}

// ---------------------------------------------------------------------------
// Logits for large batches: a 64-token x 64-expert tile per block, K in chunks
// of 32.  Each thread owns 4x4 outputs; products are chained in fp32 over one
// 32-wide chunk and the chunk sums are accumulated in fp64.
// ---------------------------------------------------------------------------
constexpr int RT_T = 64, RT_E = 64, RT_K = 32;

__global__ void __launch_bounds__(256) route_logits_tiled(const uint16_t *__restrict__ x,
                                                          int64_t T, int64_t H,
                                                          const float *__restrict__ G, int E,
                                                          double *__restrict__ part) {
    __shared__ float xs[RT_K][RT_T + 4];
    __shared__ float gs[RT_K][RT_E + 4];
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * RT_T;
    const int e0 = blockIdx.y * RT_E;
    double dacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) dacc[i][j] = 0.0;

    for (int64_t kc = 0; kc < H; kc += RT_K) {
        {   // x tile: 64 tokens x 32 bf16; thread loads 8 bf16 (16 B)
            const int tt = tid / 4, kk = (tid % 4) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t0 + tt < T) v = *reinterpret_cast<const uint4 *>(x + (t0 + tt) * H + kc + kk);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                xs[kk + 2 * i][tt] = bf16_bits_to_float(w4[i] & 0xffffu);
                xs[kk + 2 * i + 1][tt] = bf16_bits_to_float(w4[i] >> 16);
            }
        }
        {   // gate tile: 64 experts x 32 fp32; thread loads 2 float4
#pragma unroll
            for (int r = 0; r < 2; r++) {
                const int idx = tid + 256 * r;
                const int ee = idx / 8, kk = (idx % 8) * 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e0 + ee < E) v = *reinterpret_cast<const float4 *>(G + static_cast<int64_t>(e0 + ee) * H + kc + kk);
                gs[kk][ee] = v.x;
                gs[kk + 1][ee] = v.y;
                gs[kk + 2][ee] = v.z;
                gs[kk + 3][ee] = v.w;
            }
        }
        __syncthreads();
        float facc[4][4];
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int j = 0; j < 4; j++) facc[i][j] = 0.0f;
#pragma unroll 8
        for (int kk = 0; kk < RT_K; kk++) {
            const float4 xv = *reinterpret_cast<const float4 *>(&xs[kk][ty * 4]);
            const float4 gv = *reinterpret_cast<const float4 *>(&gs[kk][tx * 4]);
            const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
            const float ga[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) facc[i][j] = fmaf(xa[i], ga[j], facc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int j = 0; j < 4; j++) dacc[i][j] += static_cast<double>(facc[i][j]);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int64_t t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int e = e0 + tx * 4 + j;
            if (e < E) part[t * E + e] = dacc[i][j];
        }
    }
}

// ---------------------------------------------------------------------------
// Selection: one warp per token.
// ---------------------------------------------------------------------------
struct SelArgs {
    const double *part;
    int KS;
    int64_t T;
    const float *bias;
    int E, k, n_group, topk_group;
    float rsf, topp;
    int32_t *idx_out;
    float *w_out;
    float *gap_out;
};

// (value, index) argmax across the warp; ties go to the lower index.
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
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

__global__ void __launch_bounds__(SEL_WARPS * 32) route_select(SelArgs a) {
    extern __shared__ float smem[];
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * SEL_WARPS + wid;
    if (t >= a.T) return;
    const int E = a.E;
    float *s_sm = smem + wid * (2 * E + 64);
    float *b_sm = s_sm + E;
    float *g_sm = b_sm + E;          // group scores [<=32]
    int *pick = reinterpret_cast<int *>(g_sm + 32);  // chosen experts [<=32]

    for (int e = lane; e < E; e += 32) {
        double l = 0.0;
        for (int ks = 0; ks < a.KS; ks++) l += a.part[(static_cast<int64_t>(ks) * a.T + t) * E + e];
        const float logit = static_cast<float>(l);
        const float s = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(logit))));
        s_sm[e] = s;
        b_sm[e] = s + a.bias[e];
    }
    __syncwarp();

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

    // top-k experts of b among the kept groups, descending, ties to lower index
    float bk = 0.0f;
    for (int r = 0; r < a.k; r++) {
        float v = -INFINITY;
        int i = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            if (!((gmask >> (e / gsz)) & 1u)) continue;
            const float b = b_sm[e];
            if (b > v || (b == v && e < i)) {
                v = b;
                i = e;
            }
        }
        warp_argmax(v, i);
        if (i >= E) i = -1;  // no candidate left (only with non-finite scores)
        if (lane == 0) pick[r] = i;
        __syncwarp();
        if (i >= 0 && lane == (i & 31)) b_sm[i] = -INFINITY;  // taken
        __syncwarp();
        bk = v;
    }
    float rest = -INFINITY;
    {
        int i = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            if (!((gmask >> (e / gsz)) & 1u)) continue;
            const float b = b_sm[e];
            if (b > rest || (b == rest && e < i)) {
                rest = b;
                i = e;
            }
        }
        warp_argmax(rest, i);
    }
    const int cand = __popc(gmask) * gsz;

    if (lane == 0) {
        const int k = a.k;
        int32_t *idx = a.idx_out + t * k;
        float *w = a.w_out + t * k;
        float sum = 0.0f;
        for (int r = 0; r < k; r++)
            if (pick[r] >= 0) sum += s_sm[pick[r]];
        for (int r = 0; r < k; r++) {
            idx[r] = pick[r];
            w[r] = pick[r] >= 0 ? (s_sm[pick[r]] / sum) * a.rsf : 0.0f;
        }
        if (a.topp > 0.0f && a.topp < 1.0f) {
            // rank the slots by weight (ties keep slot order), keep the shortest
            // prefix that reaches topp * total
            float total = 0.0f;
            for (int r = 0; r < k; r++) total += w[r];
            const float target = a.topp * total;
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
        if (a.gap_out) {
            float gap = (cand > k) ? (bk - rest) : INFINITY;
            if (any_dropped) gap = fminf(gap, last_kept - best_dropped);
            a.gap_out[t] = gap;
        }
    }
}

// K-splits for the small-batch logits: slices of at most 512 columns (the
// registers a lane holds), a multiple of 4 columns each.  H % 64 == 0.
int route_ks_for(int64_t T, int64_t H) {
    if (T > 64) return 1;
    for (int64_t ks = (H + 511) / 512; ks <= H / 4; ks++)
        if (H % ks == 0 && (H / ks) % 4 == 0) return static_cast<int>(ks);
    return static_cast<int>(H / 4);
}

size_t route_part_bytes(int64_t T, int64_t H, int E) {
    return static_cast<size_t>(route_ks_for(T, H)) * static_cast<size_t>(T) * E * sizeof(double);
}

moe_status launch_route(const uint16_t *x, int64_t T, int64_t H, const float *gate,
                        const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                        float *w_out, float *gap_out, double *part, cudaStream_t stream) {
    if (T == 0) return MOE_OK;
    const int E = cfg->n_experts;
    const int KS = route_ks_for(T, H);
    if (T <= 64) {
        dim3 grid((E + 7) / 8, KS);
        route_logits_small<<<grid, 256, 0, stream>>>(x, T, H, gate, E, KS, part);
    } else {
        dim3 grid(static_cast<unsigned>((T + RT_T - 1) / RT_T), (E + RT_E - 1) / RT_E);
        route_logits_tiled<<<grid, 256, 0, stream>>>(x, T, H, gate, E, part);
    }
    SelArgs a;
    a.part = part;
    a.KS = KS;
    a.T = T;
    a.bias = bias;
    a.E = E;
    a.k = cfg->top_k;
    a.n_group = cfg->n_group;
    a.topk_group = cfg->topk_group;
    a.rsf = cfg->routed_scaling_factor;
    a.topp = cfg->expert_topp;
    a.idx_out = idx_out;
    a.w_out = w_out;
    a.gap_out = gap_out;
    const size_t smem = SEL_WARPS * (2 * E + 64) * sizeof(float);
    const unsigned grid = static_cast<unsigned>((T + SEL_WARPS - 1) / SEL_WARPS);
    route_select<<<grid, SEL_WARPS * 32, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
