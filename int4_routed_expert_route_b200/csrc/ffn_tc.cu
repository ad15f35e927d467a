// ffn_tc.cu -- expert FFN for large batches on the 5th-generation tensor cores.
//
// Batch-union grouped GEMM ("Show HN: running GLM 5.2 on a slow computer",
// implemented features: batch-union MoE, each unique expert read once and
// applied to all positions routed to it; dequant-on-use int4 weights).  Two
// passes, each a persistent kernel over tiles of 128 weight rows x <=128 tokens
// of one expert:
//   pass 1 (gate/up): D_g = Q_g X^T, D_u = Q_u X^T  (bf16 x bf16 -> fp32 in TMEM)
//                     h = silu(s_g D_g) * (s_u D_u)  -> fp16 h[pair][I]
//   pass 2 (down):    D = Q_d H^T                   (fp16 x fp16 -> fp32 in TMEM)
//                     y[t] += w_pair * s_d * D      (red.add into fp32 y)
// int4 codes are exact in bf16 and fp16, so dequantising to 16 bits adds no
// error; the row scale is applied in the epilogue in fp32.
//
// Per k-step (64 columns) of a tile: the codes of the 128 weight rows arrive
// in a 6-deep cp.async ring (32 bytes per row and matrix); the 128 threads
// convert them (thread = row) into the canonical K-major 128B-swizzled
// shared-memory layout; the token rows are gathered by cp.async straight into
// the same layout, 4 steps ahead; one thread issues tcgen05.mma (M=128, N =
// tokens rounded up to 16, K=16 x 4) and tcgen05.commit signals an mbarrier
// that gates the reuse of the buffers two steps later.  All waits are bounded:
// on timeout the kernel latches MOE_FLAG_WAIT_TIMEOUT, stops, frees its tensor
// memory and returns.
#include <cstring>

#include "common.cuh"

namespace moe {

void record_stage_event(cudaEvent_t ev, cudaStream_t s);

namespace tc {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BK = 64;        // columns per k-step (one 128-byte swizzle row)
constexpr int NT = 128;       // max tokens per tile (MMA N)
constexpr int THREADS = 128;  // 4 warps: producers, converters and epilogue
constexpr int SB = 6;         // token-tile ring depth
constexpr int PB = 4;         // token prefetch distance (steps)
constexpr int SNB = 6;        // code-staging ring depth
constexpr int PN = 5;         // code prefetch distance (steps)
constexpr int SA = 2;         // converted weight tiles (double buffer)
constexpr int NBAR = 4;       // MMA-completion barrier ring
constexpr uint32_t TMEM_COLS = 256;

constexpr int TILE_BYTES = BM * BK * 2;     // 16 KB: 128 rows x 128 B
constexpr int BTILE_BYTES = NT * BK * 2;    // 16 KB
constexpr int STAGE_NIB = BM * (BK / 2);    // 4 KB of codes per matrix per step

template <int NMAT>
struct Smem {
    static constexpr size_t a_off = 0;                                     // [SA][NMAT][TILE]
    static constexpr size_t b_off = a_off + static_cast<size_t>(SA) * NMAT * TILE_BYTES;  // [SB][BTILE]
    static constexpr size_t n_off = b_off + static_cast<size_t>(SB) * BTILE_BYTES;       // [SNB][NMAT][STAGE_NIB]
    static constexpr size_t tok_off = n_off + static_cast<size_t>(SNB) * NMAT * STAGE_NIB;  // [NT] int32
    static constexpr size_t bar_off = tok_off + NT * 4;                    // [NBAR] u64
    static constexpr size_t misc_off = bar_off + NBAR * 8;                 // tmem addr, tile id, abort
    static constexpr size_t total = misc_off + 64 + 1024;                  // + alignment slack
};

struct TcArgs {
    int64_t T, H, I;
    int32_t k, E;
    const moe_expert *experts;
    const moe_expert *shared;
    const int32_t *offsets, *tok, *tile_off, *list;
    int32_t n_shared_chunks;
    unsigned *tile_counter;
    uint32_t *flags;
    const uint16_t *x;  // pass 1 B operand (bf16 [T, H])
    __half *h;          // pass 1 output / pass 2 B operand (fp16 [T*k + T, I])
    float *y;           // pass 2 output
    const float *w;     // routing weights by pair id [T*k]
    int32_t bits;       // 4 (the tensor-core path takes int4 experts)
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait on a barrier phase; false on timeout (~ seconds).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t it = 0; it < (1u << 26); it++)
        if (mbar_try(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major, 128-byte swizzled operand tile descriptor (rows at 128 B pitch,
// 8-row groups 1024 B apart, 16-byte chunks xor-swizzled by row % 8).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);         // start address
    d |= static_cast<uint64_t>(1) << 16;                          // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;                  // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                          // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                          // SWIZZLE_128B
    return d;
}
// kind::f16 instruction descriptor: fp32 accumulate, A/B fmt (0 fp16, 1 bf16),
// both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t f16_idesc(uint32_t ab_fmt, uint32_t n) {
    return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | ((n >> 3) << 17) | ((BM >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
                 ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
                   "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
                   "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
                   "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Byte offset of 16-byte chunk c of row r inside a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// 8 int4 codes (one 32-bit word, consecutive columns) -> 8 16-bit values q
// (exact), as 4 words of value pairs.  magic = bit pattern of 16-bit 128 (bf16)
// or 1024 (fp16) in both halves; sub = the pattern of magic + 8.
__device__ __forceinline__ uint4 codes_to_16bit(uint32_t v, uint32_t magic, uint32_t sub) {
    const uint32_t lo = v & 0x0F0F0F0Fu;         // even columns, one per byte
    const uint32_t hi = (v >> 4) & 0x0F0F0F0Fu;  // odd columns
    uint32_t o[4];
#pragma unroll
    for (int m = 0; m < 4; m++) {
        const uint32_t p = __byte_perm(lo, hi, static_cast<uint32_t>(m | ((4 + m) << 8)));
        o[m] = (p & 0x00FF00FFu) | magic;
    }
    uint4 r;
    if (magic == 0x43004300u) {
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r.x) : "r"(o[0]), "r"(sub));
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r.y) : "r"(o[1]), "r"(sub));
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r.z) : "r"(o[2]), "r"(sub));
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r.w) : "r"(o[3]), "r"(sub));
    } else {
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.x) : "r"(o[0]), "r"(sub));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.y) : "r"(o[1]), "r"(sub));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.z) : "r"(o[2]), "r"(sub));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r.w) : "r"(o[3]), "r"(sub));
    }
    return r;
}

struct Tile {
    const moe_expert *ex;
    const int32_t *toks;  // nullable: identity (shared expert)
    int64_t hrow;         // first h row of the segment
    int32_t j0, n;        // token range within the segment
    int32_t m0;           // first weight row
    bool shared;
};

__device__ __forceinline__ bool decode_tile(const TcArgs &a, int64_t tile, int mtiles, Tile &t) {
    const int64_t c = tile / mtiles;
    t.m0 = static_cast<int32_t>(tile % mtiles) * BM;
    if (c < a.n_shared_chunks) {
        t.ex = a.shared;
        t.toks = nullptr;
        t.hrow = a.T * a.k;
        t.j0 = static_cast<int32_t>(c * NT);
        t.n = static_cast<int32_t>(a.T - t.j0 < NT ? a.T - t.j0 : NT);
        t.shared = true;
        return true;
    }
    const int32_t cr = static_cast<int32_t>(c - a.n_shared_chunks);
    int lo = 0, hi = a.E;  // largest e with tile_off[e] <= cr
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.tile_off[mid] <= cr) lo = mid;
        else hi = mid;
    }
    const int e = lo;
    const int o0 = a.offsets[e], o1 = a.offsets[e + 1];
    t.ex = a.experts + e;
    t.toks = a.tok + o0;
    t.hrow = o0;
    t.j0 = (cr - a.tile_off[e]) * NT;
    t.n = min(NT, o1 - o0 - t.j0);
    t.shared = false;
    return t.n > 0;
}

__device__ __forceinline__ bool qm_ok(const moe_qmat &m, int64_t rows, int64_t cols) {
    return m.q != nullptr && m.scale != nullptr && m.bits == 4 && m.rows == rows && m.cols == cols;
}

// ---------------------------------------------------------------------------
// The persistent grouped-GEMM kernel.  PASS 1: gate/up + SwiGLU, PASS 2: down.
// ---------------------------------------------------------------------------
template <int PASS>
__global__ void __launch_bounds__(THREADS, 1) tc_ffn(TcArgs a) {
    constexpr int NMAT = PASS == 1 ? 2 : 1;
    using L = Smem<NMAT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *a_tiles = sm + L::a_off;
    uint8_t *b_tiles = sm + L::b_off;
    uint8_t *nib = sm + L::n_off;
    int32_t *tok_s = reinterpret_cast<int32_t *>(sm + L::tok_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar_off);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + L::misc_off);  // [0] tmem, [1] tile, [2] abort

    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t K = PASS == 1 ? a.H : a.I;        // reduction length
    const int64_t R = PASS == 1 ? a.I : a.H;        // weight rows
    const int mtiles = static_cast<int>(R / BM);
    const int KT = static_cast<int>(K / BK);
    const int64_t rb = K / 2;                        // bytes per code row
    const uint32_t fmt = PASS == 1 ? 1u : 0u;        // bf16 (x) or fp16 (h)
    const uint32_t magic = PASS == 1 ? 0x43004300u : 0x64006400u;
    const uint32_t subv = PASS == 1 ? 0x43084308u : 0x64086408u;

    if (tid == 0) {
        for (int i = 0; i < NBAR; i++) mbar_init(smem_u32(&bars[i]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        misc[2] = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&misc[0])), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    const int64_t total_chunks = static_cast<int64_t>(a.n_shared_chunks) + a.tile_off[a.E];
    const int64_t ntiles = total_chunks * mtiles;
    uint32_t kglobal = 0;  // k-steps issued by this CTA so far (barrier phases)
    bool abort = false;

    for (;;) {
        __syncthreads();  // everyone has read the previous tile id
        if (tid == 0) misc[1] = atomicAdd(a.tile_counter, 1u);
        __syncthreads();
        const int64_t tile = misc[1];
        if (tile >= ntiles) break;
        Tile t;
        if (!decode_tile(a, tile, mtiles, t)) continue;
        const moe_qmat *mats[2];
        if (PASS == 1) {
            mats[0] = &t.ex->gate;
            mats[1] = &t.ex->up;
        } else {
            mats[0] = &t.ex->down;
            mats[1] = &t.ex->down;
        }
        const uint8_t *qm[2];
        bool ok = true;
        for (int mi = 0; mi < NMAT; mi++) {
            const moe_qmat m = *mats[mi];
            ok = ok && qm_ok(m, R, K);
            qm[mi] = m.q;
        }
        if (!ok) {
            if (tid == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
            continue;
        }
        const int npad = (t.n + 15) & ~15;
        // token / h row indices of the tile
        for (int j = tid; j < NT; j += THREADS) {
            int32_t r = 0;
            if (j < t.n) {
                if (PASS == 1) r = t.toks ? t.toks[t.j0 + j] : t.j0 + j;
                else r = static_cast<int32_t>(t.hrow + t.j0 + j);
            }
            tok_s[j] = r;
        }
        __syncthreads();

        // producers ------------------------------------------------------
        auto issue_b = [&](int kt) {  // token rows of k-step kt -> ring slot
            uint8_t *bt = b_tiles + static_cast<size_t>(kt % SB) * BTILE_BYTES;
            const uint32_t base = smem_u32(bt);
            for (int q = tid; q < npad * 8; q += THREADS) {
                const int j = q >> 3, c = q & 7;
                const bool have = j < t.n;
                const uint16_t *src;
                if (PASS == 1) src = a.x + static_cast<int64_t>(tok_s[j]) * a.H + static_cast<int64_t>(kt) * BK + c * 8;
                else src = reinterpret_cast<const uint16_t *>(a.h) + static_cast<int64_t>(tok_s[j]) * a.I + static_cast<int64_t>(kt) * BK + c * 8;
                cp_async16(base + sw_off(j, c), have ? src : reinterpret_cast<const uint16_t *>(qm[0]), have ? 16u : 0u);
            }
        };
        auto issue_n = [&](int kt) {  // codes of k-step kt -> staging slot
            uint8_t *ns = nib + static_cast<size_t>(kt % SNB) * NMAT * STAGE_NIB;
            for (int q = tid; q < NMAT * BM * 2; q += THREADS) {
                const int mi = q / (BM * 2), r = (q >> 1) % BM, half = q & 1;
                const uint8_t *src = qm[mi] + static_cast<int64_t>(t.m0 + r) * rb + static_cast<int64_t>(kt) * (BK / 2) + half * 16;
                cp_async16(smem_u32(ns + mi * STAGE_NIB + r * 32 + half * 16), src, 16u);
            }
        };
        // prologue: B(0..PB-1), N(0..PN-1) in PB commit groups (group j holds B(j))
        for (int j = 0; j < PB; j++) {
            if (j < KT) issue_b(j);
            if (j == 0)
                for (int q = 0; q <= PN - PB && q < KT; q++) issue_n(q);
            else if (j + PN - PB < KT) issue_n(j + PN - PB);
            cp_commit();
        }

        for (int kt = 0; kt < KT && !abort; kt++) {
            const uint32_t kg = kglobal + kt;
            // buffers of step kt-2 are reused below: its MMAs must be complete
            if (kt >= 2) {
                const uint32_t kp = kg - 2;
                if (!mbar_wait(smem_u32(&bars[kp % NBAR]), (kp / NBAR) & 1)) abort = true;
            }
            if (__syncthreads_or(abort)) {
                abort = true;
                break;
            }
            if (kt + PB < KT) issue_b(kt + PB);
            if (kt + PN < KT) issue_n(kt + PN);
            cp_commit();
            cp_wait<PB>();
            __syncthreads();
            // convert the codes of step kt (thread = row) into the swizzled tile
            {
                const int r = tid;
                const uint8_t *ns = nib + static_cast<size_t>(kt % SNB) * NMAT * STAGE_NIB;
                uint8_t *at = a_tiles + static_cast<size_t>(kt % SA) * NMAT * TILE_BYTES;
#pragma unroll
                for (int mi = 0; mi < NMAT; mi++) {
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(ns + mi * STAGE_NIB + r * 32);
                    const uint4 w1 = *reinterpret_cast<const uint4 *>(ns + mi * STAGE_NIB + r * 32 + 16);
                    const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint8_t *tile = at + mi * TILE_BYTES;
#pragma unroll
                    for (int c = 0; c < 8; c++)
                        *reinterpret_cast<uint4 *>(tile + sw_off(r, c)) = codes_to_16bit(wv[c], magic, subv);
                }
            }
            fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idesc = f16_idesc(fmt, static_cast<uint32_t>(npad));
                const uint32_t abase = smem_u32(a_tiles + static_cast<size_t>(kt % SA) * NMAT * TILE_BYTES);
                const uint32_t bbase = smem_u32(b_tiles + static_cast<size_t>(kt % SB) * BTILE_BYTES);
#pragma unroll
                for (int ks = 0; ks < BK / 16; ks++) {
                    const uint64_t bd = sw128_desc(bbase) + static_cast<uint64_t>(ks * 2);
#pragma unroll
                    for (int mi = 0; mi < NMAT; mi++) {
                        const uint64_t ad = sw128_desc(abase + mi * TILE_BYTES) + static_cast<uint64_t>(ks * 2);
                        mma_f16(tmem + mi * NT, ad, bd, idesc, (kt > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(smem_u32(&bars[kg % NBAR]));
            }
        }
        cp_wait_all();
        if (abort) break;
        // wait for the last k-step's MMAs (they complete in issue order)
        {
            const uint32_t kl = kglobal + KT - 1;
            if (!mbar_wait(smem_u32(&bars[kl % NBAR]), (kl / NBAR) & 1)) abort = true;
        }
        if (__syncthreads_or(abort)) {
            abort = true;
            break;
        }
        kglobal += KT;
        tc_fence_after();

        // epilogue: thread = weight row m0 + tid (TMEM lane tid)
        const int row = t.m0 + tid;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        if (PASS == 1) {
            const float sg = t.ex->gate.scale[row], su = t.ex->up.scale[row];
            bool ovf = false;
            for (int c0 = 0; c0 < npad; c0 += 32) {
                uint32_t g[32], u[32];
                tmem_ld32(lane_addr + c0, g);
                tmem_ld32(lane_addr + NT + c0, u);
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int j = c0 + i;
                    if (j < t.n) {
                        const float gv = __uint_as_float(g[i]) * sg;
                        const float uv = __uint_as_float(u[i]) * su;
                        const float hv = silu(gv) * uv;
                        ovf |= !(fabsf(hv) <= 65504.0f);
                        a.h[(t.hrow + t.j0 + j) * a.I + row] = __float2half_rn(hv);
                    }
                }
            }
            if (ovf) raise_flag(a.flags, MOE_FLAG_FP16_OVERFLOW);
        } else {
            const float sd = t.ex->down.scale[row];
            for (int c0 = 0; c0 < npad; c0 += 32) {
                uint32_t d[32];
                tmem_ld32(lane_addr + c0, d);
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int j = c0 + i;
                    if (j < t.n) {
                        const int64_t hr = t.hrow + t.j0 + j;
                        const int64_t tk = t.shared ? (t.j0 + j) : a.tok[hr];
                        const float wgt = t.shared ? 1.0f : a.w[a.list[hr]];
                        atomicAdd(a.y + tk * a.H + row, wgt * (__uint_as_float(d[i]) * sd));
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (abort && tid == 0) raise_flag(a.flags, MOE_FLAG_WAIT_TIMEOUT);
    cp_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

}  // namespace tc

bool tc_ok(int64_t H, int64_t I) {
    return H % tc::BM == 0 && I % tc::BM == 0 && H % tc::BK == 0 && I % tc::BK == 0 &&
           H / tc::BK >= 1 && I / tc::BK >= 1;
}

size_t tc_h_bytes(int64_t T, int32_t k, int64_t I) {
    return static_cast<size_t>(T * k + T) * static_cast<size_t>(I) * sizeof(__half);
}

moe_status run_tc_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k, int32_t E,
                        const moe_expert *experts, const moe_expert *shared, const int32_t *offsets,
                        const int32_t *tok, const int32_t *tile_off, const int32_t *list,
                        const float *w, void *h, float *y, unsigned *counters, uint32_t *flags,
                        cudaStream_t stream, cudaEvent_t ev_down) {
    using namespace tc;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    TcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.T = T;
    a.H = H;
    a.I = I;
    a.k = k;
    a.E = E;
    a.experts = experts;
    a.shared = shared;
    a.offsets = offsets;
    a.tok = tok;
    a.tile_off = tile_off;
    a.list = list;
    a.n_shared_chunks = shared ? static_cast<int32_t>((T + NT - 1) / NT) : 0;
    a.flags = flags;
    a.x = x;
    a.h = static_cast<__half *>(h);
    a.y = y;
    a.w = w;
    a.bits = 4;
    if (cudaMemsetAsync(counters, 0, 2 * sizeof(unsigned), stream) != cudaSuccess) return MOE_ERR_CUDA;
    {
        const size_t smem = Smem<2>::total;
        if (cudaFuncSetAttribute(tc_ffn<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        a.tile_counter = counters;
        tc_ffn<1><<<sms, THREADS, smem, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (ev_down) record_stage_event(ev_down, stream);
    {
        const size_t smem = Smem<1>::total;
        if (cudaFuncSetAttribute(tc_ffn<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        a.tile_counter = counters + 1;
        tc_ffn<2><<<sms, THREADS, smem, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace moe
