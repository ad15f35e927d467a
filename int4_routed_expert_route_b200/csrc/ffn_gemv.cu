// ffn_gemv.cu -- CUDA-core expert FFN for small batches (decode, MTP verify).
//
// The weights are streamed once per call from HBM in their packed form and
// decoded on use ("Show HN: running GLM 5.2 on a slow computer", implemented
// features: dequant-on-use, single rows kept in f32).  Each unique expert of
// the batch is read once and applied to all tokens routed to it (batch-union).
//
// Work layout.  A "segment" is one expert with its token list; an "item" is a
// tile of RT consecutive output rows of one segment.  The items of a call are
// split into equal contiguous ranges, one per block, so every block streams the
// same number of weight rows.  Inside a block, warp w owns the 16-byte chunks
// [32w, 32w+32) of every row (a K-slice): the activations of that slice live in
// registers for the whole segment, each lane issues one 128-bit streaming load
// per row and matrix, and the partial dot products are reduced with warp
// shuffles and then across the K-slice warps in shared memory (fixed order:
// the result does not depend on timing).
//
// Decoding.  A code c of b bits is placed into the mantissa of 2^23
// (float bits 0x4B000000 | c << e, exact for c << e < 2^23), and one packed
// f32x2 subtraction of 2^23 + bias * 2^e leaves q * 2^e exactly.  The
// activation of that column was multiplied by 2^-e (exact) when it was loaded,
// so one f32x2 FMA accumulates q * x.  Per int4 weight this is ~1 LOP3, 1/2
// FADD2 and 1/2 FFMA2.  The row scale is applied once to the row's sum.
#include <cstring>

#include "common.cuh"
#include "dequant.cuh"

namespace moe {

void record_stage_event(cudaEvent_t ev, cudaStream_t s);

// ---------------------------------------------------------------------------
// Arguments and segment resolution.
// ---------------------------------------------------------------------------
struct GemvArgs {
    const uint16_t *x;   // [T, H] bf16 (gate/up input)
    const float *h;      // [P_all, I] fp32 (down input)
    float *h_out;        // [P_all, I] fp32 (gate/up output)
    float *yp;           // [P_all, H] fp32 per-pair output (layer mode down)
    float *y;            // [T, H] fp32 (single mode down, accumulated)
    int64_t T, H, I;
    int32_t k, bits;
    int32_t mode;        // 0: layer (segments from the bucket), 1: one expert
    const moe_expert *experts;  // device [E]
    const moe_expert *shared;   // device, nullable
    moe_expert single;          // mode 1
    const int32_t *rows;        // mode 1: token of each row (nullable: identity)
    const float *row_w;         // mode 1: weight of each row (nullable: 1)
    int64_t n_rows;             // mode 1
    const int32_t *unique, *n_unique, *offsets, *tok;  // mode 0
    uint32_t *flags;
};

struct Seg {
    const moe_expert *ex;
    const int32_t *toks;  // token per j (nullable: j)
    int64_t n_tok;
    int64_t hrow;         // first h / yp row of the segment
};

__device__ __forceinline__ int64_t num_segments(const GemvArgs &a) {
    if (a.mode == 1) return 1;
    return static_cast<int64_t>(*a.n_unique) + (a.shared ? 1 : 0);
}

__device__ __forceinline__ Seg segment(const GemvArgs &a, int64_t s) {
    Seg g;
    if (a.mode == 1) {
        g.ex = &a.single;
        g.toks = a.rows;
        g.n_tok = a.n_rows;
        g.hrow = 0;
        return g;
    }
    const int nu = *a.n_unique;
    if (s < nu) {
        const int e = a.unique[s];
        const int o0 = a.offsets[e], o1 = a.offsets[e + 1];
        g.ex = a.experts + e;
        g.toks = a.tok + o0;
        g.n_tok = o1 - o0;
        g.hrow = o0;
    } else {
        g.ex = a.shared;
        g.toks = nullptr;
        g.n_tok = a.T;
        g.hrow = a.T * a.k;
    }
    return g;
}

__device__ __forceinline__ bool qmat_ok(const moe_qmat &m, int bits, int64_t rows, int64_t cols) {
    return m.q != nullptr && m.scale != nullptr && m.bits == bits && m.rows == rows && m.cols == cols;
}

// ---------------------------------------------------------------------------
// Gate/up + SwiGLU.   h[row_of(t)] = silu(s_g * Q_g x_t) * (s_u * Q_u x_t)
// ---------------------------------------------------------------------------
template <int BITS, int TG, int RT>
__global__ void __launch_bounds__(384) gateup_gemv(GemvArgs a) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W;            // words per lane chunk
    constexpr int PW = D::CPW / 2;                // f32x2 pairs per word
    constexpr int NP = CW * PW;                   // f32x2 activation pairs per token
    extern __shared__ float red[];                // [KW][RT][2][TG]
    const int lane = threadIdx.x & 31, kw = threadIdx.x >> 5, KW = blockDim.x >> 5;
    const int64_t H = a.H, I = a.I;
    const int64_t rb = H * BITS / 8;              // bytes per weight row
    const int64_t chunk = static_cast<int64_t>(kw) * 32 + lane;
    const bool active = chunk * D::CH < rb;
    const int64_t col0 = chunk * D::NC;           // first column of this lane
    const int64_t tiles = I / RT;
    const int64_t nseg = num_segments(a);
    const int64_t nitems = nseg * tiles;
    const int64_t i0 = nitems * blockIdx.x / gridDim.x, i1 = nitems * (blockIdx.x + 1) / gridDim.x;

    f2 xs[TG][NP];
    int64_t cur_seg = -1;
    for (int64_t item = i0; item < i1; item++) {
        const int64_t s = item / tiles;
        const int64_t r0 = (item % tiles) * RT;
        const Seg g = segment(a, s);
        const moe_qmat mg = g.ex->gate, mu = g.ex->up;
        if (!qmat_ok(mg, BITS, I, H) || !qmat_ok(mu, BITS, I, H)) {
            if (threadIdx.x == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
            continue;
        }
        for (int64_t t0 = 0; t0 < g.n_tok; t0 += TG) {
            if (s != cur_seg || g.n_tok > TG) {
#pragma unroll
                for (int t = 0; t < TG; t++) {
                    const int64_t j = t0 + t;
                    const bool have = active && j < g.n_tok;
                    const int64_t tok = have ? (g.toks ? g.toks[j] : j) : 0;
                    const uint16_t *xr = a.x + tok * H + col0;
#pragma unroll
                    for (int w = 0; w < CW; w++) {
                        // D::CPW columns per word, read as bf16 pairs
#pragma unroll
                        for (int p = 0; p < PW; p++) {
                            float v0 = 0.f, v1 = 0.f;
                            if (have) {
                                const uint32_t pr = *reinterpret_cast<const uint32_t *>(xr + w * D::CPW + 2 * p);
                                v0 = ldexpf(bf16_bits_to_float(pr & 0xffffu), -D::exp_of(2 * p));
                                v1 = ldexpf(bf16_bits_to_float(pr >> 16), -D::exp_of(2 * p + 1));
                            }
                            xs[t][w * PW + p] = f2_make(v0, v1);
                        }
                    }
                }
                cur_seg = s;
            }
            uint32_t wg[RT][CW], wu[RT][CW];
#pragma unroll
            for (int r = 0; r < RT; r++) {
                if (active) {
                    load_chunk<BITS>(mg.q + (r0 + r) * rb + chunk * D::CH, wg[r]);
                    load_chunk<BITS>(mu.q + (r0 + r) * rb + chunk * D::CH, wu[r]);
                } else {
#pragma unroll
                    for (int w = 0; w < CW; w++) wg[r][w] = wu[r][w] = 0u;
                }
            }
            f2 acc[RT][2][TG];
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int m = 0; m < 2; m++)
#pragma unroll
                    for (int t = 0; t < TG; t++) acc[r][m][t].v = 0ull;
            if (active) {
#pragma unroll
                for (int r = 0; r < RT; r++) {
#pragma unroll
                    for (int w = 0; w < CW; w++) {
                        f2 qg[PW], qu[PW];
                        D::decode(wg[r][w], qg);
                        D::decode(wu[r][w], qu);
#pragma unroll
                        for (int t = 0; t < TG; t++)
#pragma unroll
                            for (int p = 0; p < PW; p++) {
                                f2_fma(acc[r][0][t], qg[p], xs[t][w * PW + p]);
                                f2_fma(acc[r][1][t], qu[p], xs[t][w * PW + p]);
                            }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int m = 0; m < 2; m++)
#pragma unroll
                    for (int t = 0; t < TG; t++) {
                        const float v = warp_sum(f2_lo(acc[r][m][t]) + f2_hi(acc[r][m][t]));
                        if (lane == 0) red[((kw * RT + r) * 2 + m) * TG + t] = v;
                    }
            __syncthreads();
            for (int q = threadIdx.x; q < RT * TG; q += blockDim.x) {
                const int r = q / TG, t = q % TG;
                if (t0 + t < g.n_tok) {
                    float sg = 0.f, su = 0.f;
                    for (int w = 0; w < KW; w++) {
                        sg += red[((w * RT + r) * 2 + 0) * TG + t];
                        su += red[((w * RT + r) * 2 + 1) * TG + t];
                    }
                    const float gv = sg * mg.scale[r0 + r];
                    const float uv = su * mu.scale[r0 + r];
                    a.h_out[(g.hrow + t0 + t) * I + r0 + r] = silu(gv) * uv;
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// Down projection.  layer mode: yp[row_of(t)][j] = s_d[j] * Q_d[j] . h
//                   single mode: y[t][j] += row_w * s_d[j] * Q_d[j] . h
// ---------------------------------------------------------------------------
template <int BITS, int TG, int RT>
__global__ void __launch_bounds__(384) down_gemv(GemvArgs a) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W;
    constexpr int PW = D::CPW / 2;
    constexpr int NP = CW * PW;
    extern __shared__ float red[];                // [KW][RT][TG]
    const int lane = threadIdx.x & 31, kw = threadIdx.x >> 5, KW = blockDim.x >> 5;
    const int64_t H = a.H, I = a.I;
    const int64_t rb = I * BITS / 8;
    const int64_t chunk = static_cast<int64_t>(kw) * 32 + lane;
    const bool active = chunk * D::CH < rb;
    const int64_t col0 = chunk * D::NC;
    const int64_t tiles = H / RT;
    const int64_t nseg = num_segments(a);
    const int64_t nitems = nseg * tiles;
    const int64_t i0 = nitems * blockIdx.x / gridDim.x, i1 = nitems * (blockIdx.x + 1) / gridDim.x;

    f2 hs[TG][NP];
    int64_t cur_seg = -1;
    for (int64_t item = i0; item < i1; item++) {
        const int64_t s = item / tiles;
        const int64_t r0 = (item % tiles) * RT;
        const Seg g = segment(a, s);
        const moe_qmat md = g.ex->down;
        if (!qmat_ok(md, BITS, H, I)) {
            if (threadIdx.x == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
            continue;
        }
        for (int64_t t0 = 0; t0 < g.n_tok; t0 += TG) {
            if (s != cur_seg || g.n_tok > TG) {
#pragma unroll
                for (int t = 0; t < TG; t++) {
                    const int64_t j = t0 + t;
                    const bool have = active && j < g.n_tok;
                    const float *hr = a.h + (g.hrow + (have ? j : 0)) * I + col0;
#pragma unroll
                    for (int w = 0; w < CW; w++) {
#pragma unroll
                        for (int p = 0; p < PW; p++) {
                            float v0 = 0.f, v1 = 0.f;
                            if (have) {
                                const float2 pr = *reinterpret_cast<const float2 *>(hr + w * D::CPW + 2 * p);
                                v0 = ldexpf(pr.x, -D::exp_of(2 * p));
                                v1 = ldexpf(pr.y, -D::exp_of(2 * p + 1));
                            }
                            hs[t][w * PW + p] = f2_make(v0, v1);
                        }
                    }
                }
                cur_seg = s;
            }
            uint32_t wd[RT][CW];
#pragma unroll
            for (int r = 0; r < RT; r++) {
                if (active) load_chunk<BITS>(md.q + (r0 + r) * rb + chunk * D::CH, wd[r]);
                else {
#pragma unroll
                    for (int w = 0; w < CW; w++) wd[r][w] = 0u;
                }
            }
            f2 acc[RT][TG];
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int t = 0; t < TG; t++) acc[r][t].v = 0ull;
            if (active) {
#pragma unroll
                for (int r = 0; r < RT; r++)
#pragma unroll
                    for (int w = 0; w < CW; w++) {
                        f2 qd[PW];
                        D::decode(wd[r][w], qd);
#pragma unroll
                        for (int t = 0; t < TG; t++)
#pragma unroll
                            for (int p = 0; p < PW; p++) f2_fma(acc[r][t], qd[p], hs[t][w * PW + p]);
                    }
            }
#pragma unroll
            for (int r = 0; r < RT; r++)
#pragma unroll
                for (int t = 0; t < TG; t++) {
                    const float v = warp_sum(f2_lo(acc[r][t]) + f2_hi(acc[r][t]));
                    if (lane == 0) red[(kw * RT + r) * TG + t] = v;
                }
            __syncthreads();
            for (int q = threadIdx.x; q < RT * TG; q += blockDim.x) {
                const int r = q / TG, t = q % TG;
                const int64_t j = t0 + t;
                if (j < g.n_tok) {
                    float sum = 0.f;
                    for (int w = 0; w < KW; w++) sum += red[(w * RT + r) * TG + t];
                    const float v = sum * md.scale[r0 + r];
                    if (a.mode == 0) {
                        a.yp[(g.hrow + j) * H + r0 + r] = v;
                    } else {
                        const int64_t tok = g.toks ? g.toks[j] : j;
                        const float wgt = a.row_w ? a.row_w[j] : 1.0f;
                        float *yy = a.y + tok * H + r0 + r;
                        *yy = *yy + wgt * v;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// Combine: y[t] = (accumulate ? y[t] : 0) + sum_slot w * yp[pos] + yp[shared t]
// ---------------------------------------------------------------------------
__global__ void combine_kernel(float *__restrict__ y, const float *__restrict__ yp,
                               const int32_t *__restrict__ pos, const float *__restrict__ w,
                               int64_t T, int64_t H, int32_t k, int has_shared, int accumulate) {
    const int64_t n4 = T * H / 4;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = (i * 4) / H, j = (i * 4) % H;
        float4 acc = accumulate ? *reinterpret_cast<const float4 *>(y + t * H + j)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < k; s++) {
            const int q = pos[t * k + s];
            if (q < 0) continue;
            const float ws = w[t * k + s];
            const float4 v = *reinterpret_cast<const float4 *>(yp + static_cast<int64_t>(q) * H + j);
            acc.x += ws * v.x;
            acc.y += ws * v.y;
            acc.z += ws * v.z;
            acc.w += ws * v.w;
        }
        if (has_shared) {
            const float4 v = *reinterpret_cast<const float4 *>(yp + (T * k + t) * H + j);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        *reinterpret_cast<float4 *>(y + t * H + j) = acc;
    }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
constexpr int GU_RT = 4, DN_RT = 4;

template <typename K>
static int blocks_per_sm(K kern, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess) n = 1;
    return n < 1 ? 1 : n;
}

static int sm_count() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <int BITS, int TG>
static moe_status launch_gemv_bits(const GemvArgs &a, int64_t max_items_gu, int64_t max_items_dn,
                                   cudaStream_t stream, bool do_gateup, bool do_down) {
    using D = Dec<BITS>;
    const int64_t rb_gu = a.H * BITS / 8, rb_dn = a.I * BITS / 8;
    const int kw_gu = static_cast<int>((rb_gu / D::CH + 31) / 32);
    const int kw_dn = static_cast<int>((rb_dn / D::CH + 31) / 32);
    if (kw_gu > 12 || kw_dn > 12) return MOE_ERR_UNSUPPORTED;
    const int sms = sm_count();
    if (do_gateup) {
        auto kern = gateup_gemv<BITS, TG, GU_RT>;
        const int threads = kw_gu * 32;
        const size_t smem = static_cast<size_t>(kw_gu) * GU_RT * 2 * TG * sizeof(float);
        int64_t grid = static_cast<int64_t>(sms) * blocks_per_sm(kern, threads, smem);
        if (grid > max_items_gu) grid = max_items_gu;
        if (grid < 1) grid = 1;
        kern<<<static_cast<unsigned>(grid), threads, smem, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (do_down) {
        auto kern = down_gemv<BITS, TG, DN_RT>;
        const int threads = kw_dn * 32;
        const size_t smem = static_cast<size_t>(kw_dn) * DN_RT * TG * sizeof(float);
        int64_t grid = static_cast<int64_t>(sms) * blocks_per_sm(kern, threads, smem);
        if (grid > max_items_dn) grid = max_items_dn;
        if (grid < 1) grid = 1;
        kern<<<static_cast<unsigned>(grid), threads, smem, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

// Runs gate/up and/or down for the given arguments; max_segments bounds the
// number of segments (the device decides the exact count).
moe_status launch_gemv(const GemvArgs &a, int64_t max_segments, int64_t max_tok_per_seg,
                       cudaStream_t stream, bool do_gateup, bool do_down) {
    if (a.H % 64 || a.I % 64) return MOE_ERR_UNSUPPORTED;
    const int64_t mgu = max_segments * (a.I / GU_RT), mdn = max_segments * (a.H / DN_RT);
    const bool tg1 = max_tok_per_seg <= 1;
    switch (a.bits) {
    case 4: return tg1 ? launch_gemv_bits<4, 1>(a, mgu, mdn, stream, do_gateup, do_down)
                       : launch_gemv_bits<4, 2>(a, mgu, mdn, stream, do_gateup, do_down);
    case 8: return tg1 ? launch_gemv_bits<8, 1>(a, mgu, mdn, stream, do_gateup, do_down)
                       : launch_gemv_bits<8, 2>(a, mgu, mdn, stream, do_gateup, do_down);
    case 2: return launch_gemv_bits<2, 1>(a, mgu, mdn, stream, do_gateup, do_down);
    default: return MOE_ERR_INVALID_ARG;
    }
}

moe_status launch_combine(float *y, const float *yp, const int32_t *pos, const float *w,
                          int64_t T, int64_t H, int32_t k, bool has_shared, bool accumulate,
                          cudaStream_t stream) {
    const int64_t n4 = T * H / 4;
    if (n4 == 0) return MOE_OK;
    int64_t grid = (n4 + 255) / 256;
    if (grid > 4096) grid = 4096;
    combine_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(y, yp, pos, w, T, H, k,
                                                                     has_shared ? 1 : 0,
                                                                     accumulate ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe

namespace moe {

moe_status run_gemv_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k, int32_t bits,
                          const moe_expert *experts, const moe_expert *shared, const int32_t *unique,
                          const int32_t *n_unique, const int32_t *offsets, const int32_t *tok,
                          float *h, float *yp, uint32_t *flags, int64_t max_segments,
                          int64_t max_tok, cudaStream_t stream, cudaEvent_t ev_down) {
    GemvArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x;
    a.h = h;
    a.h_out = h;
    a.yp = yp;
    a.T = T;
    a.H = H;
    a.I = I;
    a.k = k;
    a.bits = bits;
    a.mode = 0;
    a.experts = experts;
    a.shared = shared;
    a.unique = unique;
    a.n_unique = n_unique;
    a.offsets = offsets;
    a.tok = tok;
    a.flags = flags;
    moe_status st = launch_gemv(a, max_segments, max_tok, stream, true, false);
    if (st != MOE_OK) return st;
    if (ev_down) record_stage_event(ev_down, stream);
    return launch_gemv(a, max_segments, max_tok, stream, false, true);
}

moe_status run_gemv_single(const uint16_t *x, int64_t T, int64_t H, int64_t I, const moe_expert &e,
                           const int32_t *rows, const float *row_w, int64_t n_rows, float *h,
                           float *y, uint32_t *flags, cudaStream_t stream) {
    GemvArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x;
    a.h = h;
    a.h_out = h;
    a.y = y;
    a.T = T;
    a.H = H;
    a.I = I;
    a.k = 1;
    a.bits = e.gate.bits;
    a.mode = 1;
    a.single = e;
    a.rows = rows;
    a.row_w = row_w;
    a.n_rows = n_rows;
    a.flags = flags;
    return launch_gemv(a, 1, n_rows, stream, true, true);
}

}  // namespace moe
