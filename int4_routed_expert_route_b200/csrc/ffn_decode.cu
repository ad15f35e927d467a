// ffn_decode.cu -- expert FFN for decode-size batches (T <= 8) on CUDA cores.
//
// Bandwidth design for HBM-bound int4 GEMV ("Show HN: running GLM 5.2 on a slow
// computer", implemented features: dequant-on-use, batch-union MoE; here the
// experts are resident in HBM instead of being streamed from disk):
//  - The rows of all unique experts of the batch (shared expert first) form one
//    row space; blocks split it so that each works inside one expert (blocks
//    per expert = grid / experts), every SM streaming about the same bytes.
//    Warp (kw, rg) owns the 16-byte chunks [32kw, 32kw+32) of the rows
//    rg, rg+RG, ... of its range; its activation slice (read with 16-byte
//    loads) stays in registers.  Each lane streams its own chunks through a
//    private cp.async ring in shared memory.
//  - int4: a lane's 32 activations become integers X = round(x * 2^F) (one
//    exponent per lane chunk, |X| < 2^22) split into three byte limbs; a code
//    word's even and odd nibbles meet the limb words in six dp4a, the code bias
//    enters as -8 * sum(X), and the chunk's dot product is exact in int32 and
//    rounded once to fp32.  int8 / int2: a code c at bit p of a word is decoded
//    as the exact float 2^23 + c*2^e (one lop3 with 0x4B000000) against
//    activations pre-scaled by 2^-e, one packed subtract and one packed FMA per
//    pair of codes.
//  - Partial dot products are reduced across the warp with a reduce-scatter
//    butterfly (V values in V-1 + log2(32/V) shuffles instead of 5V) and across
//    the K-slice warps once per run in shared memory, in a fixed order.
//  - Down: blocks write per-pair partials and count the finished rows of every
//    64-row tile of H; the block that completes a tile adds each token's
//    partials in slot order and writes y once: the weighted combine is fused
//    and deterministic (no atomics on y, no extra launch).
//  - The gate/up and down kernels launch with programmatic stream
//    serialization: each waits for its predecessor only where it reads that
//    kernel's output (down issues its weight prologue before waiting for h).
#include <cstring>

#include "common.cuh"
#include "dequant.cuh"

namespace moe {

void record_stage_event(cudaEvent_t ev, cudaStream_t s);

struct DecodeArgs {
    const uint16_t *x;  // [T, H] bf16
    int64_t T, H, I;
    int32_t k;
    const moe_expert *experts;  // device [E]
    const moe_expert *shared;   // device, nullable
    const int32_t *unique, *n_unique, *offsets, *tok, *pos, *idx;
    const float *w;   // [T, k] routing weights
    float *h;         // [T*k + T, I] fp32
    float *y;         // [T, H] fp32
    float *yp;        // [T*k + T, H] fp32 per-pair down outputs
    int32_t *tile_cnt;  // [H / 64] completion counters (zero between calls)
    int32_t accumulate;
    int32_t n_experts;
    int32_t kw, rg;   // K-slice warps, row groups (blockDim = 32 * kw * rg)
    int32_t rows_pb;  // down: max output rows per block (smem sizing)
    uint32_t *flags;
};

struct DSeg {
    const moe_expert *ex;
    const int32_t *toks;  // nullable: identity
    int64_t n_tok;
    int64_t hrow;
};

// Segments: the shared expert first when present, then the routed experts.
// With one token the routed segments are the k selection slots themselves
// (slot p is h / yp row p; a slot dropped by the expert top-p, or holding an
// index out of range, is an empty segment), read straight from the selection:
// no bucketing.  Otherwise they are the batch's unique experts in ascending
// order, with their token lists from the bucketing.
__device__ __forceinline__ int64_t dec_nseg(const DecodeArgs &a) {
    return (a.T == 1 ? static_cast<int64_t>(a.k) : static_cast<int64_t>(*a.n_unique)) + (a.shared ? 1 : 0);
}

__device__ __forceinline__ DSeg dec_seg(const DecodeArgs &a, int64_t s) {
    DSeg g;
    if (a.shared) {
        if (s == 0) {
            g.ex = a.shared;
            g.toks = nullptr;
            g.n_tok = a.T;
            g.hrow = a.T * a.k;
            return g;
        }
        s -= 1;
    }
    if (a.T == 1) {
        const int e = a.idx[s];
        const bool valid = e >= 0 && e < a.n_experts;
        if (e >= a.n_experts) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_INDEX);
        g.ex = valid ? a.experts + e : nullptr;
        g.toks = nullptr;
        g.n_tok = valid ? 1 : 0;
        g.hrow = s;
        return g;
    }
    const int e = a.unique[s];
    const int o0 = a.offsets[e], o1 = a.offsets[e + 1];
    g.ex = a.experts + e;
    g.toks = a.tok + o0;
    g.n_tok = o1 - o0;
    g.hrow = o0;
    return g;
}

// Row range [r0, r1) of this block in the union row space (nseg segments of
// seg_rows rows).  When the grid has at least one block per segment, every
// block works inside a single segment (blocks per segment = grid / nseg, the
// spare blocks idle): a block whose range straddled two experts would run two
// pipelines back to back and finish long after the others.  Otherwise equal
// contiguous ranges.
__device__ __forceinline__ void dec_block_rows(int64_t nseg, int64_t seg_rows, int64_t &r0, int64_t &r1) {
    const int64_t nb = gridDim.x, b = blockIdx.x;
    if (nseg <= 0) {
        r0 = r1 = 0;
        return;
    }
    if (nseg <= nb) {
        const int64_t bps = nb / nseg;
        const int64_t s = b / bps, piece = b % bps;
        if (s >= nseg) {
            r0 = r1 = 0;
            return;
        }
        r0 = s * seg_rows + seg_rows * piece / bps;
        r1 = s * seg_rows + seg_rows * (piece + 1) / bps;
    } else {
        const int64_t R = nseg * seg_rows;
        r0 = R * b / nb;
        r1 = R * (b + 1) / nb;
    }
}

__device__ __forceinline__ bool dqmat_ok(const moe_qmat &m, int bits, int64_t rows, int64_t cols) {
    return m.q != nullptr && m.scale != nullptr && m.bits == bits && m.rows == rows && m.cols == cols;
}

// Reduce-scatter across the warp: V values per lane in, lane keeps the full
// sum of value index bfly_index<V>(lane) in v[0].
template <int V, int OFF>
struct Bfly {
    static __device__ __forceinline__ void run(float *v, int lane) {
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < V / 2; i++) {
            const float send = upper ? v[i] : v[i + V / 2];
            const float keep = upper ? v[i + V / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
        }
        Bfly<V / 2, OFF / 2>::run(v, lane);
    }
};
template <int OFF>
struct Bfly<1, OFF> {
    static __device__ __forceinline__ void run(float *v, int lane) {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
        Bfly<1, OFF / 2>::run(v, lane);
    }
};
template <>
struct Bfly<1, 0> {
    static __device__ __forceinline__ void run(float *, int) {}
};

template <int V>
__device__ __forceinline__ int bfly_index(int lane) {
    int idx = 0, half = V / 2, off = 16;
#pragma unroll
    for (int l = 0; l < 5; l++) {
        if (half >= 1) {
            if (lane & off) idx += half;
            half >>= 1;
        }
        off >>= 1;
    }
    return idx;
}

// Lanes that write the reduced value (one per value index).
template <int V>
__device__ __forceinline__ bool bfly_writer(int lane) {
    return (lane & (32 / V - 1)) == 0;
}

// 2^-e as an exact fp32 constant (0 <= e <= 20).
__device__ __forceinline__ float exp2_neg(int e) { return __uint_as_float(static_cast<uint32_t>(127 - e) << 23); }

// Loads a lane's NC activations (contiguous, 16-byte aligned: the chunk's
// column offset is a multiple of NC) with 16-byte vector loads — every lane of
// every block reads them at the same moment, so scalar loads would queue up in
// L2 — and pre-scales them by 2^-e of their code position: f2 index w*PW + p
// holds (column w*CPW + 2p, column w*CPW + 2p + 1).
template <int BITS, typename Src>
__device__ __forceinline__ void load_act(const Src *src, bool have, f2 *out) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W, PW = D::CPW / 2, NC = CW * D::CPW;
    float v[NC];
#pragma unroll
    for (int i = 0; i < NC; i++) v[i] = 0.0f;
    if (have) {
        if constexpr (sizeof(Src) == 2) {
            static_assert(NC % 8 == 0, "bf16 activations come in 16-byte groups of 8");
#pragma unroll
            for (int i = 0; i < NC / 8; i++) {
                const uint4 q = *reinterpret_cast<const uint4 *>(src + 8 * i);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    v[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
                    v[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
                }
            }
        } else {
            static_assert(NC % 4 == 0, "fp32 activations come in 16-byte groups of 4");
#pragma unroll
            for (int i = 0; i < NC / 4; i++) {
                const float4 q = *reinterpret_cast<const float4 *>(src + 4 * i);
                v[4 * i] = q.x;
                v[4 * i + 1] = q.y;
                v[4 * i + 2] = q.z;
                v[4 * i + 3] = q.w;
            }
        }
    }
#pragma unroll
    for (int w = 0; w < CW; w++)
#pragma unroll
        for (int p = 0; p < PW; p++)
            out[w * PW + p] = f2_make(v[w * D::CPW + 2 * p] * exp2_neg(D::exp_of(2 * p)),
                                      v[w * D::CPW + 2 * p + 1] * exp2_neg(D::exp_of(2 * p + 1)));
}

// acc += decoded(chunk) . act  for one lane chunk.
template <int BITS>
__device__ __forceinline__ void chunk_fma(const uint32_t *wd, const f2 *act, f2 &acc) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W, PW = D::CPW / 2;
    if constexpr (BITS == 4) {
        const typename Dec<4>::Consts k = Dec<4>::consts();
#pragma unroll
        for (int w = 0; w < CW; w++) Dec<4>::dot(wd[w], act + w * PW, acc, k);
    } else {
#pragma unroll
        for (int w = 0; w < CW; w++) {
            f2 q[PW];
            D::decode(wd[w], q);
#pragma unroll
            for (int p = 0; p < PW; p++) f2_fma(acc, q[p], act[w * PW + p]);
        }
    }
}

// int4 dot products on the integer pipe (dp4a).  A lane's 32 activations of
// its chunk become integers X = round(x 2^F), one exponent F per lane and
// chunk with max |X| in [2^21, 2^22), split into byte limbs X = X2 2^16 +
// X1 2^8 + X0 (X0, X1 unsigned, X2 signed).  A weight word's nibbles split
// into its even and odd codes (v & 0x0F0F0F0F, (v >> 4) & 0x0F0F0F0F), each
// meeting the matching limb words in dp4a.  With the code bias folded in as
// -8 sum(X), the lane's 32-code dot product sum (c - 8) X is exact in int32
// (|.| < 32 * 8 * 2^22 = 2^30; the parts wrap modulo 2^32 on the way), and is
// rounded once to fp32 and scaled by 2^-F (exact): 9 integer instructions per
// 8 codes instead of 17 decode / f32x2 ones.  X is exact for bf16 inputs down
// to 2^-14 of the chunk's largest magnitude, and within 2^-22 of it otherwise.
struct Limbs4 {
    uint32_t e[3][4], o[3][4];  // [limb][word]: limbs of columns 8w + 0,2,4,6 / 8w + 1,3,5,7
    uint32_t bias;              // 8 * sum(X), modulo 2^32
    float inv;                  // 2^-F
};

__device__ __forceinline__ uint32_t pack_limb(int32_t a, int32_t b, int32_t c, int32_t d, int l) {
    const uint32_t sel = static_cast<uint32_t>(l | ((4 + l) << 4));
    const uint32_t ab = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), sel);
    const uint32_t cd = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), sel);
    return __byte_perm(ab, cd, 0x5410);
}

template <typename Src>
__device__ __forceinline__ void load_limbs4(const Src *src, bool have, Limbs4 &L) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = 0.0f;
    if (have) {
        if constexpr (sizeof(Src) == 2) {
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const uint4 q = *reinterpret_cast<const uint4 *>(src + 8 * i);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    v[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
                    v[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float4 q = *reinterpret_cast<const float4 *>(src + 4 * i);
                v[4 * i] = q.x;
                v[4 * i + 1] = q.y;
                v[4 * i + 2] = q.z;
                v[4 * i + 3] = q.w;
            }
        }
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i++) m = fmaxf(m, fabsf(v[i]));
    int F = 0;
    if (m > 0.0f) F = 21 - (static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127);
    F = F > 126 ? 126 : (F < -126 ? -126 : F);
    const float up = __uint_as_float(static_cast<uint32_t>(127 + F) << 23);
    L.inv = __uint_as_float(static_cast<uint32_t>(127 - F) << 23);
    int32_t X[32];
    uint32_t sum = 0u;
#pragma unroll
    for (int i = 0; i < 32; i++) {
        X[i] = __float2int_rn(v[i] * up);
        sum += static_cast<uint32_t>(X[i]);
    }
    L.bias = 8u * sum;
#pragma unroll
    for (int w = 0; w < 4; w++)
#pragma unroll
        for (int l = 0; l < 3; l++) {
            L.e[l][w] = pack_limb(X[8 * w], X[8 * w + 2], X[8 * w + 4], X[8 * w + 6], l);
            L.o[l][w] = pack_limb(X[8 * w + 1], X[8 * w + 3], X[8 * w + 5], X[8 * w + 7], l);
        }
}

// sum (c - 8) x over the lane's 32 codes (4 words), as fp32.
__device__ __forceinline__ float dot4_dp4a(const uint32_t *wd, const Limbs4 &L) {
    uint32_t a0 = 0u, a1 = 0u;
    int32_t a2 = 0;
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t ev = wd[w] & 0x0F0F0F0Fu, od = (wd[w] >> 4) & 0x0F0F0F0Fu;
        asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(a0) : "r"(ev), "r"(L.e[0][w]));
        asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(a0) : "r"(od), "r"(L.o[0][w]));
        asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(a1) : "r"(ev), "r"(L.e[1][w]));
        asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(a1) : "r"(od), "r"(L.o[1][w]));
        asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(a2) : "r"(ev), "r"(L.e[2][w]));
        asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(a2) : "r"(od), "r"(L.o[2][w]));
    }
    const uint32_t d = a0 + (a1 << 8) + (static_cast<uint32_t>(a2) << 16) - L.bias;
    return __int2float_rn(static_cast<int32_t>(d)) * L.inv;
}

// A lane's activation registers for one token: dp4a limbs for int4, pre-scaled
// fp32 pairs for the f32x2 decode of int8 / int2.
template <int BITS>
struct ActRegs {
    f2 v[Chunk<BITS>::W * (Dec<BITS>::CPW / 2)];
};
template <>
struct ActRegs<4> {
    Limbs4 L;
};

template <int BITS, typename Src>
__device__ __forceinline__ void load_act_regs(const Src *src, bool have, ActRegs<BITS> &r) {
    if constexpr (BITS == 4) load_limbs4<Src>(src, have, r.L);
    else load_act<BITS, Src>(src, have, r.v);
}

// decoded(chunk) . act of one lane chunk
template <int BITS>
__device__ __forceinline__ float chunk_dot(const uint32_t *wd, const ActRegs<BITS> &r) {
    if constexpr (BITS == 4) {
        return dot4_dp4a(wd, r.L);
    } else {
        f2 acc;
        acc.v = 0ull;
        chunk_fma<BITS>(wd, r.v, acc);
        return f2_sum(acc);
    }
}

// Per-lane asynchronous copy ring.  Every lane prefetches exactly the chunks it
// will consume into its own shared-memory slots (cp.async), S-1 steps ahead, and
// waits only for its own copy groups: no barrier is needed, and the prefetch
// depth no longer costs registers.
template <int CH>
__device__ __forceinline__ void cp_async_chunk(void *smem_dst, const void *gsrc) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    if constexpr (CH == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int BITS>
__device__ __forceinline__ void lds_chunk(const uint8_t *p, uint32_t w[Chunk<BITS>::W]) {
    if constexpr (Chunk<BITS>::W == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        w[0] = v.x; w[1] = v.y;
    }
}

constexpr int DEC_RMAX = 128;  // rows per run (shared-memory partials)
constexpr int GU_S = 2;        // gate/up copy-ring stages (of GU_U rows)
constexpr int DN_S = 4;        // down copy-ring stages (of DN_U rows)
constexpr int DN_RMAX = 512;   // rows per down run

// ---------------------------------------------------------------------------
// Gate/up + SwiGLU
// ---------------------------------------------------------------------------
template <int BITS, int TG, int U>
__global__ void __launch_bounds__(384, 1) gateup_decode(DecodeArgs a) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W;
    constexpr int V = U * 2 * TG;
    extern __shared__ __align__(16) uint8_t dsm_gu[];
    float *red = reinterpret_cast<float *>(dsm_gu);  // [DEC_RMAX][2][TG][KW]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t *ring_base = dsm_gu + static_cast<size_t>(DEC_RMAX) * 2 * TG * a.kw * sizeof(float);
    const int KW = a.kw, RG = a.rg;
    const int kw = warp % KW, rg = warp / KW;
    const int64_t H = a.H, I = a.I;
    const int64_t rb = H * BITS / 8;
    const int64_t chunk = static_cast<int64_t>(kw) * 32 + lane;
    const bool active = chunk * D::CH < rb;
    const int64_t col0 = chunk * D::NC;
    // One token: its activations and the block's rows are known before the
    // routing is (every expert sees token 0; the segments are the shared
    // expert and the k routed slots), so the activations load while the router
    // still runs, and the shared expert's blocks do all their work then.
    ActRegs<BITS> xs[TG];
    int64_t xs_seg = -1;
    const bool one_token = a.T == 1;
    int64_t r0, r1;
    if (one_token) {
        dec_block_rows(dec_nseg(a), I, r0, r1);
        load_act_regs<BITS, uint16_t>(a.x + col0, active, xs[0]);
        if (!(a.shared && r0 < r1 && r1 <= I)) griddep_wait();  // routing of this batch
    } else {
        griddep_wait();
        dec_block_rows(dec_nseg(a), I, r0, r1);
    }
    griddep_launch();  // the down kernel may start its weight prologue

    for (int64_t r = r0; r < r1;) {
        const int64_t s = r / I;
        const int64_t run_end = min(r1, (s + 1) * I);
        const int64_t i_begin = r - s * I;
        const DSeg g = dec_seg(a, s);
        if (!g.ex) {  // an empty slot
            r = run_end;
            continue;
        }
        const moe_qmat mg = g.ex->gate, mu = g.ex->up;
        const bool ok = dqmat_ok(mg, BITS, I, H) && dqmat_ok(mu, BITS, I, H);
        if (!ok && threadIdx.x == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
        for (int64_t sub = 0; ok && sub < run_end - r; sub += DEC_RMAX) {
            const int m = static_cast<int>(run_end - r - sub < DEC_RMAX ? run_end - r - sub : DEC_RMAX);
            const int64_t ib = i_begin + sub;  // first row (within the expert) of this sub-run
            for (int64_t t0 = 0; t0 < g.n_tok; t0 += TG) {
                const int nmy = rg < m ? (m - rg + RG - 1) / RG : 0;
                const int nsteps = (nmy + U - 1) / U;
                uint8_t *ring = ring_base + static_cast<size_t>(warp) * (GU_S * U * 2 * 32 * D::CH);
                auto issue = [&](int step) {
                    if (step < nsteps) {
                        uint8_t *st = ring + static_cast<size_t>(step % GU_S) * (U * 2 * 32 * D::CH);
#pragma unroll
                        for (int u = 0; u < U; u++) {
                            const int lr = rg + RG * (step * U + u);
                            if (active && lr < m) {
                                const int64_t row = ib + lr;
                                cp_async_chunk<D::CH>(st + ((u * 2 + 0) * 32 + lane) * D::CH, mg.q + row * rb + chunk * D::CH);
                                cp_async_chunk<D::CH>(st + ((u * 2 + 1) * 32 + lane) * D::CH, mu.q + row * rb + chunk * D::CH);
                            }
                        }
                    }
                    cp_async_commit();
                };
#pragma unroll
                for (int st = 0; st < GU_S - 1; st++) issue(st);  // weights first, then the activations
                if (!one_token && (xs_seg != s || g.n_tok > TG)) {
#pragma unroll
                    for (int t = 0; t < TG; t++) {
                        const bool have = active && t0 + t < g.n_tok;
                        const int64_t tok = have ? (g.toks ? g.toks[t0 + t] : t0 + t) : 0;
                        load_act_regs<BITS, uint16_t>(a.x + tok * H + col0, have, xs[t]);
                    }
                    xs_seg = s;
                }
                // the epilogue's row scales, loaded while the rows stream
                float pre_g = 0.0f, pre_u = 0.0f;
                if (static_cast<int>(threadIdx.x) < m * TG) {
                    const int64_t row = ib + threadIdx.x / TG;
                    pre_g = mg.scale[row];
                    pre_u = mu.scale[row];
                }
                for (int st = 0; st < nsteps; st++) {
                    issue(st + GU_S - 1);
                    cp_async_wait<GU_S - 1>();
                    const uint8_t *sl = ring + static_cast<size_t>(st % GU_S) * (U * 2 * 32 * D::CH);
                    uint32_t wr[U][2][CW];
#pragma unroll
                    for (int u = 0; u < U; u++)
#pragma unroll
                        for (int mm = 0; mm < 2; mm++) lds_chunk<BITS>(sl + ((u * 2 + mm) * 32 + lane) * D::CH, wr[u][mm]);
                    float v[V];
#pragma unroll
                    for (int u = 0; u < U; u++)
#pragma unroll
                        for (int mm = 0; mm < 2; mm++)
#pragma unroll
                            for (int t = 0; t < TG; t++)
                                v[(u * 2 + mm) * TG + t] = active ? chunk_dot<BITS>(wr[u][mm], xs[t]) : 0.0f;
                    Bfly<V, 16>::run(v, lane);
                    if (bfly_writer<V>(lane)) {
                        const int idx = bfly_index<V>(lane);
                        const int u = idx / (2 * TG), mm = (idx / TG) % 2, t = idx % TG;
                        const int lr = rg + RG * (st * U + u);
                        if (lr < m) red[((lr * 2 + mm) * TG + t) * KW + kw] = v[0];
                    }
                }
                cp_async_wait_all();
                __syncthreads();
                for (int q = threadIdx.x; q < m * TG; q += blockDim.x) {
                    const int lr = q / TG, t = q % TG;
                    if (t0 + t < g.n_tok) {
                        float sg = 0.f, su = 0.f;
                        for (int w = 0; w < KW; w++) {
                            sg += red[((lr * 2 + 0) * TG + t) * KW + w];
                            su += red[((lr * 2 + 1) * TG + t) * KW + w];
                        }
                        const int64_t row = ib + lr;
                        const bool pre = q == static_cast<int>(threadIdx.x);
                        const float gv = sg * (pre ? pre_g : mg.scale[row]), uv = su * (pre ? pre_u : mu.scale[row]);
                        a.h[(g.hrow + t0 + t) * I + row] = silu(gv) * uv;
                    }
                }
                __syncthreads();
            }
        }
        r = run_end;
    }
}

// ---------------------------------------------------------------------------
// Down projection with the weighted combine fused.
// Rows of all unique experts' down matrices form one row space split in equal
// contiguous ranges (as for gate/up).  A block writes the unweighted per-pair
// outputs yp[pair][j] = s_d[j] * (Q_d[j] . h_pair) of its rows, then counts the
// rows it finished in every 64-row tile of H it touched; the block that
// completes a tile (all segments done) combines it: y[t][j] = (y) +
// sum_slot w * yp[pos(t,slot)][j] + yp[shared t][j], in slot order.
// ---------------------------------------------------------------------------
constexpr int DN_TILE = 64;
constexpr int kMaxTiles = 768;  // counters live in the 4 KiB workspace header

template <int BITS, int TG, int U>
__global__ void __launch_bounds__(TG == 1 ? 512 : 384, 1) down_decode(DecodeArgs a) {
    using D = Dec<BITS>;
    constexpr int CW = Chunk<BITS>::W;
    constexpr int V = U * TG;
    extern __shared__ __align__(16) uint8_t dsm_dn[];
    float *red = reinterpret_cast<float *>(dsm_dn);  // [DN_RMAX][TG][KW]
    uint8_t *ring_base = dsm_dn + static_cast<size_t>(DN_RMAX) * TG * a.kw * sizeof(float);
    __shared__ int my_tiles[DN_RMAX / DN_TILE + 1];
    __shared__ int n_my_tiles;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int KW = a.kw, RG = a.rg;
    const int kw = warp % KW, rg = warp / KW;
    const int64_t H = a.H, I = a.I, T = a.T;
    const int64_t rb = I * BITS / 8;
    const int64_t chunk = static_cast<int64_t>(kw) * 32 + lane;
    const bool active = chunk * D::CH < rb;
    const int64_t col0 = chunk * D::NC;
    const int64_t nseg = dec_nseg(a);
    int64_t r0, r1;
    dec_block_rows(nseg, H, r0, r1);
    // routing slots of the batch, staged once (T * k <= 8 * 32)
    __shared__ int32_t s_pos[8 * 32];
    __shared__ float s_w[8 * 32];
    for (int i = threadIdx.x; i < T * a.k; i += blockDim.x) {
        // one token: slot p is row p unless dropped (see dec_seg)
        s_pos[i] = T == 1 ? (a.idx[i] >= 0 && a.idx[i] < a.n_experts ? i : -1) : a.pos[i];
        s_w[i] = a.w[i];
    }

    ActRegs<BITS> hs[TG];
    bool h_ready = false;  // h comes from the gate/up kernel: wait before the first read
    for (int64_t r = r0; r < r1;) {
        const int64_t s = r / H;
        const int64_t run_end = min(r1, (s + 1) * H);
        const int64_t j_begin = r - s * H;
        const DSeg g = dec_seg(a, s);
        const moe_qmat md = g.ex ? g.ex->down : moe_qmat{};
        const bool ok = !g.ex || dqmat_ok(md, BITS, H, I);  // an empty slot computes nothing but counts its rows
        if (!ok && threadIdx.x == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
        for (int64_t sub = 0; sub < run_end - r; sub += DN_RMAX) {
            const int m = static_cast<int>(run_end - r - sub < DN_RMAX ? run_end - r - sub : DN_RMAX);
            const int64_t jb = j_begin + sub;
            for (int64_t t0 = 0; ok && t0 < g.n_tok; t0 += TG) {
                const int nmy = rg < m ? (m - rg + RG - 1) / RG : 0;
                const int nsteps = (nmy + U - 1) / U;
                uint8_t *ring = ring_base + static_cast<size_t>(warp) * (DN_S * U * 32 * D::CH);
                auto issue = [&](int step) {
                    if (step < nsteps) {
                        uint8_t *st = ring + static_cast<size_t>(step % DN_S) * (U * 32 * D::CH);
#pragma unroll
                        for (int u = 0; u < U; u++) {
                            const int lr = rg + RG * (step * U + u);
                            if (active && lr < m)
                                cp_async_chunk<D::CH>(st + (u * 32 + lane) * D::CH, md.q + (jb + lr) * rb + chunk * D::CH);
                        }
                    }
                    cp_async_commit();
                };
#pragma unroll
                for (int st = 0; st < DN_S - 1; st++) issue(st);
                if (!h_ready) {
                    griddep_wait();
                    h_ready = true;
                }
                float pre_s = 0.0f;  // the epilogue's row scale, loaded while the rows stream
                if (static_cast<int>(threadIdx.x) < m * TG) pre_s = md.scale[jb + threadIdx.x / TG];
#pragma unroll
                for (int t = 0; t < TG; t++) {
                    const bool have = active && t0 + t < g.n_tok;
                    load_act_regs<BITS, float>(a.h + (g.hrow + (have ? t0 + t : 0)) * I + col0, have, hs[t]);
                }
                for (int st = 0; st < nsteps; st++) {
                    issue(st + DN_S - 1);
                    cp_async_wait<DN_S - 1>();
                    const uint8_t *sl = ring + static_cast<size_t>(st % DN_S) * (U * 32 * D::CH);
                    uint32_t wr[U][CW];
#pragma unroll
                    for (int u = 0; u < U; u++) lds_chunk<BITS>(sl + (u * 32 + lane) * D::CH, wr[u]);
                    float v[V];
#pragma unroll
                    for (int u = 0; u < U; u++)
#pragma unroll
                        for (int t = 0; t < TG; t++) v[u * TG + t] = active ? chunk_dot<BITS>(wr[u], hs[t]) : 0.0f;
                    Bfly<V, 16>::run(v, lane);
                    if (bfly_writer<V>(lane)) {
                        const int idx = bfly_index<V>(lane);
                        const int u = idx / TG, t = idx % TG;
                        const int lr = rg + RG * (st * U + u);
                        if (lr < m) red[(lr * TG + t) * KW + kw] = v[0];
                    }
                }
                cp_async_wait_all();
                __syncthreads();
                for (int q = threadIdx.x; q < m * TG; q += blockDim.x) {
                    const int lr = q / TG, t = q % TG;
                    if (t0 + t < g.n_tok) {
                        float d = 0.f;
                        for (int w = 0; w < KW; w++) d += red[(lr * TG + t) * KW + w];
                        const int64_t j = jb + lr;
                        a.yp[(g.hrow + t0 + t) * H + j] = d * (q == static_cast<int>(threadIdx.x) ? pre_s : md.scale[j]);
                    }
                }
                __syncthreads();
            }
            // completion accounting for the 64-row tiles this sub-run touched
            // (one thread per tile, all atomics in flight together)
            __threadfence();
            if (threadIdx.x == 0) n_my_tiles = 0;
            __syncthreads();
            {
                const int64_t ja = jb, je = jb + m;
                const int64_t c = ja / DN_TILE + threadIdx.x;
                if (c * DN_TILE < je) {
                    const int64_t lo = c * DN_TILE > ja ? c * DN_TILE : ja;
                    const int64_t hi = (c + 1) * DN_TILE < je ? (c + 1) * DN_TILE : je;
                    const int add = static_cast<int>(hi - lo);
                    const int need = static_cast<int>(nseg * DN_TILE);
                    const int old = atomicAdd(a.tile_cnt + c, add);
                    if (old + add == need) my_tiles[atomicAdd(&n_my_tiles, 1)] = static_cast<int>(c);
                }
            }
            __syncthreads();
            const int nt = n_my_tiles;
            if (nt > 0) __threadfence();
            // combine every tile this sub-run completed in one pass (independent loads)
            for (int64_t q = threadIdx.x; q < static_cast<int64_t>(nt) * DN_TILE * T; q += blockDim.x) {
                const int64_t c = my_tiles[q / (DN_TILE * T)];
                const int64_t rem = q % (DN_TILE * T);
                const int64_t t = rem / DN_TILE;
                const int64_t j = c * DN_TILE + rem % DN_TILE;
                float acc = a.accumulate ? a.y[t * H + j] : 0.0f;
                const float sh = a.shared ? __ldcg(a.yp + (T * a.k + t) * H + j) : 0.0f;
#pragma unroll 8
                for (int sl = 0; sl < a.k; sl++) {
                    const int p = s_pos[t * a.k + sl];
                    const float v = p >= 0 ? __ldcg(a.yp + static_cast<int64_t>(p) * H + j) : 0.0f;
                    acc += s_w[t * a.k + sl] * v;
                }
                acc += sh;
                a.y[t * H + j] = acc;
            }
            if (threadIdx.x < nt) a.tile_cnt[my_tiles[threadIdx.x]] = 0;
        }
        r = run_end;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int dec_sm_count() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

static constexpr int GU_U = 8, DN_U = 4;  // rows per ring stage

bool decode_ok(int64_t T, int64_t H, int64_t I, int32_t k, int32_t bits) {
    (void)k;
    if (T < 1 || T > 8 || H % 64 || I % 64 || H / DN_TILE > kMaxTiles) return false;
    const int ch = bits == 2 ? 8 : 16;
    const int64_t kw_gu = (H * bits / 8 / ch + 31) / 32, kw_dn = (I * bits / 8 / ch + 31) / 32;
    return kw_gu <= 12 && kw_dn <= 12;
}

template <int BITS, int TG>
static moe_status launch_decode_bits(DecodeArgs a, cudaStream_t stream, cudaEvent_t ev_down) {
    using D = Dec<BITS>;
    const int sms = dec_sm_count();
    const int64_t rb_gu = a.H * BITS / 8, rb_dn = a.I * BITS / 8;
    const int kw_gu = static_cast<int>((rb_gu / D::CH + 31) / 32);
    const int kw_dn = static_cast<int>((rb_dn / D::CH + 31) / 32);
    {
        DecodeArgs g = a;
        g.kw = kw_gu;
        g.rg = 12 / kw_gu > 0 ? 12 / kw_gu : 1;
        const int threads = 32 * g.kw * g.rg;
        const size_t smem = static_cast<size_t>(DEC_RMAX) * 2 * TG * g.kw * sizeof(float) +
                            static_cast<size_t>(threads / 32) * GU_S * GU_U * 2 * 32 * D::CH;
        auto kern = gateup_decode<BITS, TG, GU_U>;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (launch_pdl(kern, dim3(sms), dim3(threads), smem, stream, g) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (ev_down) record_stage_event(ev_down, stream);
    {
        DecodeArgs d = a;
        d.kw = kw_dn;
        const int dn_warps = TG == 1 ? 16 : 12;  // 16 warps at T = 1 (128 registers suffice there)
        d.rg = dn_warps / kw_dn > 0 ? dn_warps / kw_dn : 1;
        const int threads = 32 * d.kw * d.rg;
        const size_t smem = static_cast<size_t>(DN_RMAX) * TG * d.kw * sizeof(float) +
                            static_cast<size_t>(threads / 32) * DN_S * DN_U * 32 * D::CH;
        auto kern = down_decode<BITS, TG, DN_U>;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (launch_pdl(kern, dim3(sms), dim3(threads), smem, stream, d) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

moe_status run_decode_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k,
                            int32_t bits, const moe_expert *experts, int32_t n_experts, const moe_expert *shared,
                            const int32_t *unique, const int32_t *n_unique, const int32_t *offsets,
                            const int32_t *tok, const int32_t *pos, const int32_t *idx,
                            const float *w, float *h, float *yp, int32_t *tile_cnt, float *y,
                            int32_t accumulate, uint32_t *flags, cudaStream_t stream,
                            cudaEvent_t ev_down) {
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x = x;
    a.T = T;
    a.H = H;
    a.I = I;
    a.k = k;
    a.experts = experts;
    a.shared = shared;
    a.unique = unique;
    a.n_unique = n_unique;
    a.offsets = offsets;
    a.tok = tok;
    a.pos = pos;
    a.idx = idx;
    a.w = w;
    a.h = h;
    a.y = y;
    a.yp = yp;
    a.tile_cnt = tile_cnt;
    a.accumulate = accumulate;
    a.flags = flags;
    a.n_experts = n_experts;
    const bool tg1 = T == 1;
    switch (bits) {
    case 4: return tg1 ? launch_decode_bits<4, 1>(a, stream, ev_down) : launch_decode_bits<4, 2>(a, stream, ev_down);
    case 8: return tg1 ? launch_decode_bits<8, 1>(a, stream, ev_down) : launch_decode_bits<8, 2>(a, stream, ev_down);
    case 2: return launch_decode_bits<2, 1>(a, stream, ev_down);
    default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace moe
