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
#include "select.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits for small batches: one block per expert, its 8 warps split the hidden
// dimension; exact bf16*fp32 products are accumulated in fp64, the 8 slice
// sums are added in a fixed order and the total is rounded once to fp32.
// logits[t][e] (fp32).  T <= 64.
// ---------------------------------------------------------------------------
constexpr int RL_WARPS = 8;
constexpr int RL_MAXT = 64;

__device__ __forceinline__ double dot4(float4 g, uint2 xv, double acc) {
    acc = fma(static_cast<double>(g.x), static_cast<double>(bf16_bits_to_float(xv.x & 0xffffu)), acc);
    acc = fma(static_cast<double>(g.y), static_cast<double>(bf16_bits_to_float(xv.x >> 16)), acc);
    acc = fma(static_cast<double>(g.z), static_cast<double>(bf16_bits_to_float(xv.y & 0xffffu)), acc);
    acc = fma(static_cast<double>(g.w), static_cast<double>(bf16_bits_to_float(xv.y >> 16)), acc);
    return acc;
}

// Block-level body: computes the logits of expert e = blockIdx.x for tokens
// t < T and returns them in lg[t] (valid in threads t < T).  Each lane issues
// all the gate loads of a batch of RL_NB float4 chunks before any FMA, so a
// warp has RL_NB cold HBM requests in flight instead of one.
constexpr int RL_NB = 8;

__device__ void logits_one_expert(const uint16_t *__restrict__ x, int64_t T, int64_t H,
                                  const float *__restrict__ G, double *red /* [RL_WARPS][RL_MAXT] smem */,
                                  float *lg /* [RL_MAXT] smem */) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int e = blockIdx.x;
    const int64_t L = H / RL_WARPS;  // H % 32 == 0 -> L % 4 == 0 (16-byte gate chunks)
    const int64_t k0 = static_cast<int64_t>(wid) * L;
    const float *gr = G + static_cast<int64_t>(e) * H + k0;
    for (int64_t t0 = 0; t0 < T; t0 += 4) {
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        for (int64_t jb = 4 * lane; jb < L; jb += 128 * RL_NB) {
            float4 g[RL_NB];
#pragma unroll
            for (int b = 0; b < RL_NB; b++) {
                const int64_t j = jb + 128 * b;
                g[b] = j < L ? __ldcs(reinterpret_cast<const float4 *>(gr + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                if (t0 + u < T) {
                    uint2 xv[RL_NB];
#pragma unroll
                    for (int b = 0; b < RL_NB; b++) {
                        const int64_t j = jb + 128 * b;
                        xv[b] = j < L ? *reinterpret_cast<const uint2 *>(x + (t0 + u) * H + k0 + j) : make_uint2(0u, 0u);
                    }
#pragma unroll
                    for (int b = 0; b < RL_NB; b++)
                        if (jb + 128 * b < L) acc[u] = dot4(g[b], xv[b], acc[u]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const double v = warp_sum(acc[u]);
            if (lane == 0 && t0 + u < T) red[wid * RL_MAXT + t0 + u] = v;
        }
    }
    __syncthreads();
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
        double v = 0.0;
        for (int w = 0; w < RL_WARPS; w++) v += red[w * RL_MAXT + t];
        lg[t] = static_cast<float>(v);
    }
}

__global__ void __launch_bounds__(RL_WARPS * 32) route_logits_small(const uint16_t *__restrict__ x,
                                                                    int64_t T, int64_t H,
                                                                    const float *__restrict__ G,
                                                                    int E, float *__restrict__ logits) {
    __shared__ double red[RL_WARPS * RL_MAXT];
    __shared__ float lg[RL_MAXT];
    logits_one_expert(x, T, H, G, red, lg);
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) logits[t * E + blockIdx.x] = lg[t];
}

// ---------------------------------------------------------------------------
// Logits for large batches: a 64-token x 64-expert tile per block, K in chunks
// of 32.  Each thread owns 4x4 outputs; products are chained in fp32 over one
// 32-wide chunk and the chunk sums are accumulated in fp64.  The chunks are
// double-buffered in shared memory: the next chunk's global loads are in
// flight while the current one is multiplied (H is a multiple of 64, so every
// chunk is full).
// ---------------------------------------------------------------------------
constexpr int RT_T = 64, RT_E = 64, RT_K = 32;

__global__ void __launch_bounds__(256) route_logits_tiled(const uint16_t *__restrict__ x,
                                                          int64_t T, int64_t H,
                                                          const float *__restrict__ G, int E,
                                                          float *__restrict__ logits) {
    __shared__ float xs[2][RT_K][RT_T + 4];
    __shared__ float gs[2][RT_K][RT_E + 4];
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * RT_T;
    const int e0 = blockIdx.y * RT_E;
    // this thread's share of a chunk: 8 bf16 of one token (16 B), 2 x 4 fp32 of the gate
    const int xt = tid / 4, xk = (tid % 4) * 8;
    const bool x_in = t0 + xt < T;
    const uint16_t *xrow = x + (x_in ? t0 + xt : 0) * H + xk;
    int g_e[2], g_k[2];
    bool g_in[2];
    const float *grow[2];
#pragma unroll
    for (int r = 0; r < 2; r++) {
        const int idx = tid + 256 * r;
        g_e[r] = idx / 8;
        g_k[r] = (idx % 8) * 4;
        g_in[r] = e0 + g_e[r] < E;
        grow[r] = G + static_cast<int64_t>(g_in[r] ? e0 + g_e[r] : 0) * H + g_k[r];
    }
    uint4 xv_r;
    float4 gv_r[2];
    auto load_chunk = [&](int64_t kc) {
        xv_r = x_in ? *reinterpret_cast<const uint4 *>(xrow + kc) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < 2; r++)
            gv_r[r] = g_in[r] ? *reinterpret_cast<const float4 *>(grow[r] + kc) : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto store_chunk = [&](int b) {
        const uint32_t w4[4] = {xv_r.x, xv_r.y, xv_r.z, xv_r.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            xs[b][xk + 2 * i][xt] = bf16_bits_to_float(w4[i] & 0xffffu);
            xs[b][xk + 2 * i + 1][xt] = bf16_bits_to_float(w4[i] >> 16);
        }
#pragma unroll
        for (int r = 0; r < 2; r++) {
            gs[b][g_k[r]][g_e[r]] = gv_r[r].x;
            gs[b][g_k[r] + 1][g_e[r]] = gv_r[r].y;
            gs[b][g_k[r] + 2][g_e[r]] = gv_r[r].z;
            gs[b][g_k[r] + 3][g_e[r]] = gv_r[r].w;
        }
    };
    double dacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) dacc[i][j] = 0.0;

    const int64_t nchunks = H / RT_K;
    load_chunk(0);
    store_chunk(0);
    __syncthreads();
    for (int64_t c = 0; c < nchunks; c++) {
        const int b = static_cast<int>(c & 1);
        if (c + 1 < nchunks) load_chunk((c + 1) * RT_K);
        float facc[4][4];
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int j = 0; j < 4; j++) facc[i][j] = 0.0f;
#pragma unroll 8
        for (int kk = 0; kk < RT_K; kk++) {
            const float4 xv = *reinterpret_cast<const float4 *>(&xs[b][kk][ty * 4]);
            const float4 gv = *reinterpret_cast<const float4 *>(&gs[b][kk][tx * 4]);
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
        // the other buffer was last read before the previous barrier
        if (c + 1 < nchunks) store_chunk(b ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int64_t t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int e = e0 + tx * 4 + j;
            if (e < E) logits[t * E + e] = static_cast<float>(dacc[i][j]);
        }
    }
}

// Routes token t with one warp; wsm is this warp's shared scratch of
// (2E + 64) floats.
__device__ void select_token(const SelArgs &a, int64_t t, float *wsm) {
    const int lane = threadIdx.x & 31;
    const int E = a.E;
    float *s_sm = wsm;
    float *b_sm = s_sm + E;
    int *pick = reinterpret_cast<int *>(b_sm + E + 32);
    for (int e = lane; e < E; e += 32) {
        const float sc = sigmoid_score(__ldcg(a.logits + t * E + e));
        s_sm[e] = sc;
        b_sm[e] = sc + a.bias[e];
    }
    __syncwarp();
    select_core(a, t, s_sm, b_sm, pick);
}

__global__ void __launch_bounds__(SEL_WARPS * 32) route_select(SelArgs a) {
    extern __shared__ float smem[];
    const int wid = threadIdx.x >> 5;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * SEL_WARPS + wid;
    if (t >= a.T) return;
    select_token(a, t, smem + wid * (2 * a.E + 64));
}

// ---------------------------------------------------------------------------
// Decode-size batches (T <= 8): logits, selection and batch-union bucketing in
// one launch.  Every block computes one expert's logits; the last block to
// finish (ticket counter in the workspace header) routes the tokens with all
// its threads (select_tokens) and then, for two or more tokens, buckets the
// (token, slot) pairs with a stable counting sort (one token's slots are its
// segments as they are).
// The counter is reset by that block for the next call.
// ---------------------------------------------------------------------------
constexpr int FUSED_MAXT = 8;

struct FusedRouteArgs {
    const uint16_t *x;
    int64_t H;
    const float *G;
    float *logits;
    SelArgs sel;
    unsigned *counter;
    int32_t *counts, *offsets, *list, *tok, *pos, *unique, *n_unique;
    uint32_t *flags;
    int32_t *zero_cnt;  // counters of the following kernels, cleared here
    int32_t n_zero;
};

// Stable bucketing of a small batch (P = T * k <= 256 pairs) by one block:
// every quantity is a direct count over the pairs (no scans over E).  The
// same outputs as the counting sort: list sorted by (expert, pair), tok, pos
// (-1 for dropped slots), counts, offsets [E+1], ascending unique experts.
// sm: 2 * P ints.
__device__ void bucket_tiny(const int32_t *idx_s, int32_t *idx_g, int P, int k, int E, int32_t *counts,
                            int32_t *offsets, int32_t *list, int32_t *tok, int32_t *pos, int32_t *unique,
                            int32_t *n_unique, uint32_t *flags, int *sm) {
    int *pe = sm;         // [P] expert of each pair, -1 if dropped or invalid
    int *first = sm + P;  // [P] pair is the first of its expert
    const int tid = threadIdx.x;
    bool bad = false;
    for (int p = tid; p < P; p += blockDim.x) {
        int e = idx_s[p];
        idx_g[p] = e;
        if (e >= E) {
            bad = true;
            e = -1;
        }
        pe[p] = e;
    }
    if (__syncthreads_or(bad) && tid == 0) raise_flag(flags, MOE_FLAG_BAD_EXPERT_INDEX);
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = pe[p];
        int f = e >= 0;
        for (int j = 0; j < p && f; j++) f = pe[j] != e;
        first[p] = f;
    }
    __syncthreads();
    for (int e = tid; e <= E; e += blockDim.x) {
        int c = 0, lt = 0;
        for (int j = 0; j < P; j++) {
            const int ej = pe[j];
            c += ej == e;
            lt += ej >= 0 && ej < e;
        }
        if (e < E) counts[e] = c;
        offsets[e] = lt;
    }
    for (int p = tid; p < P; p += blockDim.x) {
        const int e = pe[p];
        if (e < 0) {
            pos[p] = -1;
            continue;
        }
        int q = 0, u = 0;
        for (int j = 0; j < P; j++) {
            const int ej = pe[j];
            q += ej >= 0 && (ej < e || (ej == e && j < p));
            u += first[j] && ej < e;
        }
        list[q] = p;
        tok[q] = p / k;
        pos[p] = q;
        if (first[p]) unique[u] = e;
    }
    if (tid == 0) {
        int nu = 0;
        for (int j = 0; j < P; j++) nu += first[j];
        *n_unique = nu;
    }
}

__global__ void __launch_bounds__(RL_WARPS * 32) route_fused_small(FusedRouteArgs a) {
    extern __shared__ float dsm[];
    __shared__ double red[RL_WARPS * RL_MAXT];
    __shared__ float lg[RL_MAXT];
    __shared__ unsigned ticket;
    const int E = a.sel.E;
    const int64_t T = a.sel.T;
    griddep_launch();  // the gate/up kernel's blocks may be scheduled meanwhile
    // 1. this block's expert: logits, sigmoid scores and biased scores of all tokens
    logits_one_expert(a.x, T, a.H, a.G, red, lg);
    float *s_g = a.logits;          // scores [T][E]
    float *b_g = a.logits + T * E;  // biased scores [T][E]
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
        const float sc = sigmoid_score(lg[t]);
        s_g[t * E + blockIdx.x] = sc;
        b_g[t * E + blockIdx.x] = sc + a.sel.bias[blockIdx.x];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) ticket = atomicAdd(a.counter, 1u);
    __syncthreads();
    if (ticket != gridDim.x - 1) return;
    // 2. the last block: group-limited top-k of every token (all its threads at
    //    once), then bucketing
    __threadfence();
    float *s_all = dsm;               // [T][E]
    float *b_all = dsm + T * E;       // [T][E]
    for (int64_t i = threadIdx.x; i < T * E; i += blockDim.x) {
        s_all[i] = __ldcg(s_g + i);
        b_all[i] = __ldcg(b_g + i);
    }
    __syncthreads();
    const int ng = a.sel.n_group, tkg = a.sel.topk_group, k = a.sel.k;
    float *scratch = b_all + T * E;
    int32_t *idx_s = reinterpret_cast<int32_t *>(scratch + T * select_scratch_words(E, k, ng, tkg));  // [T][k]
    float *w_s = reinterpret_cast<float *>(idx_s + T * k);  // [T][k]: the top-p ranking reads it back
    select_tokens<BlockBar>(s_all, b_all, static_cast<int>(T), E, k, ng, tkg, a.sel.rsf, a.sel.topp, scratch,
                            idx_s, w_s, threadIdx.x, blockDim.x);
    for (int p = threadIdx.x; p < T * k; p += blockDim.x) a.sel.w_out[p] = w_s[p];
    if (T == 1) {  // one token: the GEMV kernels read the selection slots directly
        for (int p = threadIdx.x; p < k; p += blockDim.x) a.sel.idx_out[p] = idx_s[p];
    } else {
        bucket_tiny(idx_s, a.sel.idx_out, static_cast<int>(T * k), k, E, a.counts, a.offsets, a.list, a.tok,
                    a.pos, a.unique, a.n_unique, a.flags, reinterpret_cast<int *>(dsm));
    }
    for (int i = threadIdx.x; i < a.n_zero; i += blockDim.x) a.zero_cnt[i] = 0;
    if (threadIdx.x == 0) *a.counter = 0u;
}

// Scratch of the router: fp32 logits [T][E]; the fused small-batch router
// keeps scores and biased scores there instead ([2][T][E]).
size_t route_part_bytes(int64_t T, int64_t H, int E) {
    (void)H;
    return static_cast<size_t>(T) * E * sizeof(float) * (T <= FUSED_MAXT ? 2 : 1);
}

int route_ks_for(int64_t T, int64_t H) {
    (void)T;
    (void)H;
    return 1;
}

static SelArgs sel_args(int64_t T, const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                        float *w_out, float *gap_out, const float *logits) {
    SelArgs a;
    a.logits = logits;
    a.T = T;
    a.bias = bias;
    a.E = cfg->n_experts;
    a.k = cfg->top_k;
    a.n_group = cfg->n_group;
    a.topk_group = cfg->topk_group;
    a.rsf = cfg->routed_scaling_factor;
    a.topp = cfg->expert_topp;
    a.idx_out = idx_out;
    a.w_out = w_out;
    a.gap_out = gap_out;
    return a;
}

static size_t sel_smem(int E, int warps) { return static_cast<size_t>(warps) * (2 * E + 64) * sizeof(float); }

moe_status launch_route(const uint16_t *x, int64_t T, int64_t H, const float *gate,
                        const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                        float *w_out, float *gap_out, double *scratch, cudaStream_t stream) {
    if (T == 0) return MOE_OK;
    const int E = cfg->n_experts;
    float *logits = reinterpret_cast<float *>(scratch);
    if (T <= RL_MAXT && H % 32 == 0) {
        route_logits_small<<<E, RL_WARPS * 32, 0, stream>>>(x, T, H, gate, E, logits);
    } else {
        dim3 grid(static_cast<unsigned>((T + RT_T - 1) / RT_T), (E + RT_E - 1) / RT_E);
        route_logits_tiled<<<grid, 256, 0, stream>>>(x, T, H, gate, E, logits);
    }
    const SelArgs a = sel_args(T, bias, cfg, idx_out, w_out, gap_out, logits);
    const size_t smem = sel_smem(E, SEL_WARPS);
    const unsigned grid = static_cast<unsigned>((T + SEL_WARPS - 1) / SEL_WARPS);
    route_select<<<grid, SEL_WARPS * 32, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

bool route_fused_ok(int64_t T, int64_t H) { return T >= 1 && T <= FUSED_MAXT && H % 32 == 0; }

moe_status launch_route_fused(const uint16_t *x, int64_t T, int64_t H, const float *gate,
                              const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                              float *w_out, float *logits, unsigned *counter, int32_t *counts,
                              int32_t *offsets, int32_t *list, int32_t *tok, int32_t *pos,
                              int32_t *unique, int32_t *n_unique, uint32_t *flags,
                              int32_t *zero_cnt, int32_t n_zero, cudaStream_t stream) {
    FusedRouteArgs a;
    a.x = x;
    a.H = H;
    a.G = gate;
    a.logits = logits;
    a.sel = sel_args(T, bias, cfg, idx_out, w_out, nullptr, logits);
    a.counter = counter;
    a.counts = counts;
    a.offsets = offsets;
    a.list = list;
    a.tok = tok;
    a.pos = pos;
    a.unique = unique;
    a.n_unique = n_unique;
    a.flags = flags;
    a.zero_cnt = zero_cnt;
    a.n_zero = n_zero;
    const int E = cfg->n_experts;
    // scores, biased scores, the selection's scratch and the selected indices and weights
    size_t smem = static_cast<size_t>(
                      2 * T * E + T * (select_scratch_words(E, cfg->top_k, cfg->n_group, cfg->topk_group) + 2 * cfg->top_k)) *
                  sizeof(float);
    const size_t bsm = static_cast<size_t>(2 * T * cfg->top_k) * sizeof(int);  // bucket_tiny
    if (bsm > smem) smem = bsm;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_fused_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_fused_small<<<E, RL_WARPS * 32, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
