// ffn_tc.cu -- expert FFN for large batches on the 5th-generation tensor cores.
//
// Batch-union grouped GEMM ("Show HN: running GLM 5.2 on a slow computer",
// implemented features: batch-union MoE, each unique expert read once and
// applied to all positions routed to it; dequant-on-use int4 weights).  Two
// passes, each a persistent kernel over tiles of 128 weight rows x <=192 tokens
// of one expert:
//   pass 1 (gate/up): D_g = Q_g X^T, D_u = Q_u X^T  (bf16 x bf16 -> fp32 in TMEM)
//                     h = silu(s_g D_g) * (s_u D_u)  -> fp16 h[pair][I]
//   pass 2 (down):    D = Q_d H^T                   (fp16 x fp16 -> fp32 in TMEM)
//                     yp[pair] = s_d * D            (fp32 per-pair partials; the
//                     combine kernel adds them per token in slot order)
// int4 codes are exact in bf16 and fp16, so dequantising to 16 bits adds no
// error; the row scale is applied in the epilogue in fp32.
//
// Warp roles (pass 1: 576 threads, pass 2: 448; one CTA per SM):
//   warp 0     TMA producer: per k-step, 2D tiled loads of 64-row boxes bring the
//              tile's token rows x 64 columns of the B operand into the K-major
//              128B-swizzled layout (pass 1 reads the expert-sorted copy of x,
//              pass 2 reads h); only as many boxes as the tile has tokens
//   warp 1     MMA issuer: tcgen05.mma kind::f16, M=128, N=tokens (mult. of 16),
//              A operand from tensor memory, B from shared memory
//   warps 2-9  converters: each thread owns one weight row and one matrix (pass
//              1: gate or up) or one half of each k-step (pass 2); it streams its
//              int4 codes through a private cp.async ring, converts them to
//              16-bit values in registers ahead of time, and writes them into
//              the A stage in tensor memory (tcgen05.st) once the MMA has
//              released that stage
//   warps 10-  epilogue (pass 1: 8 warps, two per lane quarter taking alternate
//              32-column chunks; pass 2: 4): after a tile's last MMA, read the
//              accumulator lanes (tcgen05.ld), apply row scales, SwiGLU (pass 1)
//              and store
// Tensor memory (512 columns): pass 1 = gate and up accumulators (2 x 192) +
// two A stages of 2 x 32 columns; pass 2 = two accumulators (2 x 192, so the
// epilogue of one tile overlaps the MMAs of the next) + four A stages of 32.
// Hand-offs use mbarriers only; every wait is bounded (by the workspace's wait
// bound, two seconds by default) and a timeout latches MOE_FLAG_WAIT_TIMEOUT and
// stops the CTA: its TMA loads and MMAs in flight are drained with the full
// two-second bound, then it frees its tensor memory and returns.
#include <cstring>

#include <cuda.h>

#include "common.cuh"

namespace moe {

void record_stage_event(cudaEvent_t ev, cudaStream_t s);

namespace tc {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BK = 64;        // columns per k-step (one 128-byte swizzle row)
constexpr int NT = 192;       // max tokens per tile (MMA N)
constexpr int BOX = 64;       // token rows per TMA box
// producer, MMA, 8 converter warps, then the epilogue warps: pass 1 (SwiGLU on
// two accumulators, one of them to drain before the next tile) 8, pass 2 4
constexpr int threads_of(int pass) { return pass == 1 ? 576 : 448; }
constexpr int NCONV = 256;    // converter threads
constexpr int nepi_of(int pass) { return threads_of(pass) - 320; }  // epilogue threads
constexpr int SB = 4;         // token-tile ring depth

constexpr int BTILE_BYTES = NT * BK * 2;    // 24 KB: 192 rows x 128 B
constexpr int BOX_BYTES = BOX * BK * 2;     // 8 KB

template <int NMAT>
struct Smem {
    static constexpr int NACC = NMAT == 1 ? 2 : 1;   // accumulator buffers
    static constexpr int SA = NMAT == 1 ? 4 : 2;     // A stages in tensor memory
    static constexpr uint32_t a_col = NACC * NMAT * NT;          // first A column (384)
    static constexpr uint32_t a_stage_cols = NMAT * (BK / 2);    // 32-bit columns per A stage
    static constexpr uint32_t tmem_cols = 512;
    static_assert(a_col + SA * a_stage_cols <= tmem_cols, "tensor memory budget");
    static constexpr int CB = NMAT == 2 ? 32 : 16;   // code bytes (= A columns) per converter thread per k-step
    static constexpr int SC = 8;   // per-thread code ring depth (prefetch SC-1 k-steps; 12 / 16 measured no faster)
    static_assert(2 * CB == static_cast<int>(a_stage_cols), "two converter groups fill one A stage");
    static constexpr size_t b_off = 0;                                               // [SB][BTILE]
    static constexpr size_t c_off = b_off + static_cast<size_t>(SB) * BTILE_BYTES;   // [SC][CB/16][NCONV][16]
    static constexpr size_t c_stage = static_cast<size_t>(CB) * NCONV;
    static constexpr size_t bar_off = c_off + SC * c_stage;                          // barriers
    static constexpr size_t misc_off = bar_off + 24 * 8;                             // tmem addr, abort
    static_assert(2 * SB + 2 * SA + 2 * NACC + 1 <= 24, "barrier area");
    static constexpr size_t total = misc_off + 64 + 1024;                            // + alignment slack
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
    float *yp;          // pass 2 output: per-pair partials [T*k + T, H], rows as h
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
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait on a barrier phase: false once limit_ns have passed (the
// workspace's wait bound for waits on other warps' progress, kFullWaitNs for the
// drains before exit), or after 2^30 polls, whichever comes first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 28); it++) {
        for (int i = 0; i < 4; i++)
            if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// Warp-wide bounded wait: lane 0 polls, the other lanes take its result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane, uint64_t limit_ns) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, limit_ns);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
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
// Same with the A operand read from tensor memory (column address a_tmem,
// lane 0): rows of A on the 128 lanes, two 16-bit K elements per column.
__device__ __forceinline__ void mma_f16_ta(uint32_t tmem_d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
                 ::"r"(tmem_d), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
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

// Store 32 (16) consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                   "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                   "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
                   "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
                   "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                   "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                   "r"(r[14]), "r"(r[15])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// K order of the tensor-core operands.  Within every group of 8 consecutive
// K indices (one 32-bit word of codes) the MMA's K positions 2m and 2m + 1 hold
// the columns m and m + 4 (m = 0..3): once the word's even and odd nibbles are
// spread over bytes (two masks), such a pair sits in bytes 0 and 2 or 1 and 3
// of one of the two words, and one byte permute with the magic's high byte
// makes the 16-bit pair.  The B operands are stored in the same order (the
// gathered x rows of pass 1, the h rows written by pass 1's epilogue), so every
// product meets its own activation.
__device__ __forceinline__ int k_slot(int col) {  // MMA K position of column col
    const int q = col & 7;
    return (col & ~7) | (q < 4 ? 2 * q : 2 * q - 7);
}

// 8 int4 codes (one 32-bit word, consecutive columns) -> 8 16-bit values q
// (exact) in the K order above, as 4 words of value pairs (m, m + 4).
// magic = bit pattern of 16-bit 128 (bf16) or 1024 (fp16) in both halves;
// sub = the pattern of magic + 8.
__device__ __forceinline__ uint4 codes_to_16bit(uint32_t v, uint32_t magic, uint32_t sub) {
    const uint32_t even = v & 0x0F0F0F0Fu;         // bytes: nibbles 0, 2, 4, 6
    const uint32_t odd = (v >> 4) & 0x0F0F0F0Fu;   // bytes: nibbles 1, 3, 5, 7
    const uint32_t hi = (magic >> 8 & 0xFFu) * 0x01010101u;  // the magic's high byte, four times
    uint32_t o[4];
    o[0] = __byte_perm(even, hi, 0x4240);  // nibbles 0, 4
    o[1] = __byte_perm(odd, hi, 0x4240);   // 1, 5
    o[2] = __byte_perm(even, hi, 0x4341);  // 2, 6
    o[3] = __byte_perm(odd, hi, 0x4341);   // 3, 7
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
// Barrier, TMA and tensor-map helpers of the warp-specialized kernel.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, uint32_t bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

struct TcMaps {
    CUtensorMap b_main;    // pass 1: expert-sorted x; pass 2: h
    CUtensorMap b_shared;  // pass 1: x (shared expert rows); pass 2: unused (copy of b_main)
};

// Per-tile facts every role derives identically.
struct TileInfo {
    bool ok;
    Tile t;
    int npad;
    int32_t brow;                // first B row of the TMA box
    const uint8_t *q[2];         // code matrices
};

template <int PASS>
__device__ __forceinline__ TileInfo tile_info(const TcArgs &a, int64_t tile, int mtiles, int64_t R, int64_t K) {
    TileInfo ti;
    ti.ok = decode_tile(a, tile, mtiles, ti.t);
    if (!ti.ok) return ti;
    if (PASS == 1) {
        const moe_qmat g = ti.t.ex->gate, u = ti.t.ex->up;
        ti.ok = qm_ok(g, R, K) && qm_ok(u, R, K);
        ti.q[0] = g.q;
        ti.q[1] = u.q;
        ti.brow = ti.t.shared ? ti.t.j0 : static_cast<int32_t>(ti.t.hrow + ti.t.j0);
    } else {
        const moe_qmat d = ti.t.ex->down;
        ti.ok = qm_ok(d, R, K);
        ti.q[0] = d.q;
        ti.q[1] = d.q;
        ti.brow = static_cast<int32_t>(ti.t.hrow + ti.t.j0);
    }
    ti.npad = (ti.t.n + 15) & ~15;
    return ti;
}

// ---------------------------------------------------------------------------
// The warp-specialized persistent grouped-GEMM kernel.
// ---------------------------------------------------------------------------
template <int PASS>
__global__ void __launch_bounds__(threads_of(PASS), 1) tc_ffn(const __grid_constant__ TcMaps maps, TcArgs a) {
    constexpr int NMAT = PASS == 1 ? 2 : 1;
    using L = Smem<NMAT>;
    constexpr int NACC = L::NACC, SA = L::SA, CB = L::CB, SC = L::SC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *b_tiles = sm + L::b_off;
    uint8_t *cstage = sm + L::c_off;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::bar_off);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + L::misc_off);  // [0] tmem, [1] abort
    const uint32_t B_FULL = smem_u32(&bars[0]);                          // [SB]
    const uint32_t B_EMPTY = smem_u32(&bars[SB]);                        // [SB]
    const uint32_t A_FULL = smem_u32(&bars[2 * SB]);                     // [SA]
    const uint32_t A_EMPTY = smem_u32(&bars[2 * SB + SA]);               // [SA]
    const uint32_t ACC_FULL = smem_u32(&bars[2 * SB + 2 * SA]);          // [NACC]
    const uint32_t ACC_EMPTY = smem_u32(&bars[2 * SB + 2 * SA + NACC]);  // [NACC]
    const uint32_t FIN = smem_u32(&bars[2 * SB + 2 * SA + 2 * NACC]);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t K = PASS == 1 ? a.H : a.I;
    const int64_t R = PASS == 1 ? a.I : a.H;
    const int mtiles = static_cast<int>(R / BM);
    const int KT = static_cast<int>(K / BK);
    const int64_t rb = K / 2;

    if (tid == 0) {
        for (int i = 0; i < SB; i++) {
            mbar_init(B_FULL + 8 * i, 1);
            mbar_init(B_EMPTY + 8 * i, 1);
        }
        for (int i = 0; i < SA; i++) {
            mbar_init(A_FULL + 8 * i, NCONV / 32);  // one arrival per converter warp
            mbar_init(A_EMPTY + 8 * i, 1);
        }
        for (int i = 0; i < NACC; i++) {
            mbar_init(ACC_FULL + 8 * i, 1);
            mbar_init(ACC_EMPTY + 8 * i, nepi_of(PASS) / 32);  // one arrival per epilogue warp
        }
        mbar_init(FIN, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        misc[1] = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&misc[0])), "r"(L::tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    volatile uint32_t *abort_flag = &misc[1];
    const uint64_t lim = wait_limit_ns(a.flags);  // waits on the other warps' progress

    const int64_t total_chunks = static_cast<int64_t>(a.n_shared_chunks) + a.tile_off[a.E];
    const int64_t ntiles = total_chunks * mtiles;
    auto fail = [&]() {
        atomicOr(const_cast<uint32_t *>(abort_flag), 1u);
        raise_flag(a.flags, MOE_FLAG_WAIT_TIMEOUT);
    };
    // warp-uniform view of the abort flag (keeps .sync.aligned ops converged)
    auto aborted = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0u) != 0; };

    if (warp == 0) {
        // ---------------- TMA producer (one lane) ----------------
        if (lane == 0) {
            uint32_t kc = 0;  // loads issued so far
            for (int64_t tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                const TileInfo ti = tile_info<PASS>(a, tile, mtiles, R, K);
                if (!ti.ok) continue;
                const CUtensorMap *map = (PASS == 1 && ti.t.shared) ? &maps.b_shared : &maps.b_main;
                const int nbox = (ti.npad + BOX - 1) / BOX;
                const uint32_t tx = static_cast<uint32_t>(nbox * BOX_BYTES);
                bool ok = true;
                for (int kt = 0; kt < KT; kt++) {
                    const uint32_t slot = kc % SB;
                    if (!mbar_wait(B_EMPTY + 8 * slot, ((kc / SB) & 1) ^ 1, lim)) {
                        fail();
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(B_FULL + 8 * slot, tx);
                    const uint32_t dst = smem_u32(b_tiles + static_cast<size_t>(slot) * BTILE_BYTES);
                    for (int bx = 0; bx < nbox; bx++)
                        tma_load_2d(dst + bx * BOX_BYTES, map, kt * BK, ti.brow + bx * BOX, B_FULL + 8 * slot);
                    kc++;
                }
                if (!ok) break;
            }
            // drain: the last load issued into each slot has landed before exit
            // (full bound: the loads need nothing but memory)
            for (uint32_t j = kc > SB ? kc - SB : 0; j < kc; j++)
                if (!mbar_wait(B_FULL + 8 * (j % SB), (j / SB) & 1, kFullWaitNs))
                    raise_flag(a.flags, MOE_FLAG_WAIT_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (one lane) ----------------
        // The issuing thread's own instruction latency bounds back-to-back
        // MMA issue, so its k-loop is unrolled over the ring period (4 k-steps):
        // stage indices and most phase parities become compile-time, and every
        // MMA operand is a loop-invariant base plus an immediate.
        const uint32_t fmt = PASS == 1 ? 1u : 0u;
        const uint64_t bdesc0 = sw128_desc(smem_u32(b_tiles));
        const uint32_t a_tm = tmem + L::a_col;
        static_assert(SB == 4 && (SA == 2 || SA == 4), "unrolled issue assumes a 4-step ring period");
        if (lane == 0) {
            uint32_t kc = 0, tc = 0;
            for (int64_t tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                const TileInfo ti = tile_info<PASS>(a, tile, mtiles, R, K);
                if (!ti.ok) continue;
                const uint32_t idesc = f16_idesc(fmt, static_cast<uint32_t>(ti.npad));
                const uint32_t ab = tc % NACC;
                const uint32_t dbase = tmem + ab * NMAT * NT;
                if (!mbar_wait(ACC_EMPTY + 8 * ab, ((tc / NACC) & 1) ^ 1, lim)) {
                    fail();
                    break;
                }
                bool ok = true;
                if ((KT & 3) == 0 && (kc & 3) == 0) {
                    for (int kt0 = 0; kt0 < KT && ok; kt0 += 4, kc += 4) {
                        const uint32_t pb = (kc >> 2) & 1;  // phase parity of this block's B (and 4-stage A) uses
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            const uint32_t as = u % SA;
                            const uint32_t pa = SA == 4 ? pb : static_cast<uint32_t>((u >> 1) & 1);
                            if (!mbar_wait(A_FULL + 8 * as, pa, lim) || !mbar_wait(B_FULL + 8 * u, pb, lim)) {
                                fail();
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t acc0 = (kt0 + u) > 0 ? 1u : 0u;
#pragma unroll
                            for (int ks = 0; ks < BK / 16; ks++)
#pragma unroll
                                for (int mi = 0; mi < NMAT; mi++)
                                    mma_f16_ta(dbase + mi * NT, a_tm + as * L::a_stage_cols + mi * (BK / 2) + ks * 8,
                                               bdesc0 + static_cast<uint64_t>(u * (BTILE_BYTES >> 4) + ks * 2), idesc,
                                               ks > 0 ? 1u : acc0);
                            mma_commit(B_EMPTY + 8 * u);
                            mma_commit(A_EMPTY + 8 * as);
                        }
                    }
                } else {
                    // generic path (k-step counts that are not a multiple of 4)
                    for (int kt = 0; kt < KT; kt++, kc++) {
                        const uint32_t bs = kc % SB, as = kc % SA;
                        if (!mbar_wait(A_FULL + 8 * as, (kc / SA) & 1, lim) ||
                            !mbar_wait(B_FULL + 8 * bs, (kc / SB) & 1, lim)) {
                            fail();
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t bd = bdesc0 + static_cast<uint64_t>(bs * (BTILE_BYTES >> 4));
                        const uint32_t acc0 = kt > 0 ? 1u : 0u;
#pragma unroll
                        for (int ks = 0; ks < BK / 16; ks++)
#pragma unroll
                            for (int mi = 0; mi < NMAT; mi++)
                                mma_f16_ta(dbase + mi * NT, a_tm + as * L::a_stage_cols + mi * (BK / 2) + ks * 8,
                                           bd + static_cast<uint64_t>(ks * 2), idesc, ks > 0 ? 1u : acc0);
                        mma_commit(B_EMPTY + 8 * bs);
                        mma_commit(A_EMPTY + 8 * as);
                    }
                }
                if (!ok) break;
                mma_commit(ACC_FULL + 8 * ab);
                tc++;
            }
            // every MMA this thread issued has completed before the TMEM is freed
            // (full bound: issued MMAs need nothing from the other warps)
            mma_commit(FIN);
            if (!mbar_wait(FIN, 0, kFullWaitNs)) raise_flag(a.flags, MOE_FLAG_WAIT_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < 10) {
        // ---------------- converters ----------------
        const int ct = tid - 64;                 // 0..255
        const int quarter = warp & 3;            // TMEM lane quarter this warp may write
        const int grp = (warp - 2) >> 2;         // pass 1: matrix (gate, up); pass 2: k-step half
        const int r = quarter * 32 + lane;       // weight row within the tile
        const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t magic = PASS == 1 ? 0x43004300u : 0x64006400u;
        const uint32_t subv = PASS == 1 ? 0x43084308u : 0x64086408u;
        // Code prefetch cursor: runs SC-1 k-steps ahead of the conversion,
        // across tile boundaries, through this CTA's sequence of valid tiles.
        int64_t pf_tile = blockIdx.x;
        int pf_kt = 0;
        TileInfo pf;
        pf.ok = false;
        auto pf_seek = [&]() {
            for (; pf_tile < ntiles; pf_tile += gridDim.x) {
                pf = tile_info<PASS>(a, pf_tile, mtiles, R, K);
                if (pf.ok) return;
                if (ct == 0 && pf.t.n > 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_SHAPE);
            }
        };
        auto pf_issue = [&](uint32_t slot) {
            if (pf_tile < ntiles) {
                uint8_t *st = cstage + static_cast<size_t>(slot) * L::c_stage;
                const uint8_t *src = (PASS == 1 && grp ? pf.q[1] : pf.q[0]) + static_cast<int64_t>(pf.t.m0 + r) * rb +
                                     static_cast<int64_t>(pf_kt) * (BK / 2) + (PASS == 1 ? 0 : grp * 16);
#pragma unroll
                for (int hf = 0; hf < CB / 16; hf++)
                    cp_async16(smem_u32(st + (hf * NCONV + ct) * 16), src + hf * 16, 16u);
                if (++pf_kt == KT) {
                    pf_kt = 0;
                    pf_tile += gridDim.x;
                    pf_seek();
                }
            }
            cp_commit();
        };
        pf_seek();
        uint32_t kc = 0;
        for (int j = 0; j < SC - 1; j++) pf_issue(static_cast<uint32_t>(j));
        for (int64_t tile = blockIdx.x; tile < ntiles && !aborted(); tile += gridDim.x) {
            const TileInfo ti = tile_info<PASS>(a, tile, mtiles, R, K);
            if (!ti.ok) continue;
            for (int kt = 0; kt < KT && !aborted(); kt++, kc++) {
                pf_issue((kc + SC - 1) % SC);
                cp_wait<SC - 1>();
                const uint8_t *st = cstage + static_cast<size_t>(kc % SC) * L::c_stage;
                uint32_t v[CB];  // 16-bit value pairs (2 codes per byte, 2 values per column)
#pragma unroll
                for (int hf = 0; hf < CB / 16; hf++) {
                    const uint4 wq = *reinterpret_cast<const uint4 *>(st + (hf * NCONV + ct) * 16);
                    const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        const uint4 o = codes_to_16bit(wv[c], magic, subv);
                        v[hf * 16 + c * 4 + 0] = o.x;
                        v[hf * 16 + c * 4 + 1] = o.y;
                        v[hf * 16 + c * 4 + 2] = o.z;
                        v[hf * 16 + c * 4 + 3] = o.w;
                    }
                }
                const uint32_t as = kc % SA;
                // one lane polls, the warp follows; one arrival per warp
                if (!warp_wait(A_EMPTY + 8 * as, ((kc / SA) & 1) ^ 1, lane, lim)) fail();
                tc_fence_after();
                const uint32_t col = L::a_col + as * L::a_stage_cols + grp * CB;
                if constexpr (CB == 32) tmem_st32(tmem + lane_bits + col, v);
                else tmem_st16(tmem + lane_bits + col, v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(A_FULL + 8 * as);
            }
        }
        cp_wait_all();
    } else {
        // ---------------- epilogue ----------------
        const int quarter = warp & 3;                  // TMEM lane quarter this warp may read
        constexpr int CSTEP = nepi_of(PASS) / 4;      // two warps per lane quarter in pass 1: alternate chunks
        const int c_first = ((warp - 10) >> 2) * 32;   // this warp's 32-column chunks: c_first, + CSTEP, ...
        const int r = quarter * 32 + lane;             // weight row within the tile
        uint32_t tc = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles && !aborted(); tile += gridDim.x) {
            const TileInfo ti = tile_info<PASS>(a, tile, mtiles, R, K);
            if (!ti.ok) continue;
            const uint32_t ab = tc % NACC;
            if (!warp_wait(ACC_FULL + 8 * ab, (tc / NACC) & 1, lane, lim)) fail();
            tc_fence_after();
            const Tile &t = ti.t;
            const int row = t.m0 + r;
            const uint32_t lane_addr = tmem + ab * NMAT * NT + (static_cast<uint32_t>(quarter * 32) << 16);
            if (!aborted()) {
                if (PASS == 1) {
                    const float sg = t.ex->gate.scale[row], su = t.ex->up.scale[row];
                    __half *hp = a.h + (t.hrow + t.j0) * a.I + k_slot(row);  // pass 2's K order
                    bool ovf = false;
                    for (int c0 = c_first; c0 < ti.npad; c0 += CSTEP) {
                        uint32_t g[32], u[32];
                        tmem_ld32(lane_addr + c0, g);
                        tmem_ld32(lane_addr + NT + c0, u);
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const int j = c0 + i;
                            if (j < t.n) {
                                const float gv = __uint_as_float(g[i]) * sg;
                                const float uv = __uint_as_float(u[i]) * su;
                                const float hv = silu_fast(gv) * uv;
                                ovf |= !(fabsf(hv) <= 65504.0f);
                                hp[static_cast<int64_t>(j) * a.I] = __float2half_rn(hv);
                            }
                        }
                    }
                    if (ovf) raise_flag(a.flags, MOE_FLAG_FP16_OVERFLOW);
                } else {
                    const float sd = t.ex->down.scale[row];
                    float *yq = a.yp + (t.hrow + t.j0) * a.H + row;
                    for (int c0 = c_first; c0 < ti.npad; c0 += CSTEP) {
                        uint32_t d[32];
                        tmem_ld32(lane_addr + c0, d);
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const int j = c0 + i;
                            if (j < t.n) yq[static_cast<int64_t>(j) * a.H] = __uint_as_float(d[i]) * sd;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ACC_EMPTY + 8 * ab);
            tc++;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::tmem_cols) : "memory");
}

// Pass 1's B rows in the MMA's K order (k_slot): xs[q] = x[tok[q]] for the
// routed pairs q < n_rows (of cap rows), then xs[cap + t] = x[t] for the shared
// expert's T rows.  A 16-byte vector is one group of 8 columns (c0..c7) and
// becomes (c0, c4, c1, c5, c2, c6, c3, c7).
__global__ void gather_rows(const uint16_t *__restrict__ x, const int32_t *__restrict__ tok,
                            const int32_t *__restrict__ n_rows, int64_t cap, int64_t T_shared, int64_t H,
                            uint16_t *__restrict__ xs) {
    const int64_t n = *n_rows;
    const int64_t per = H / 8;  // 16-byte vectors per row
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < (cap + T_shared) * per;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t q = i / per, v = i % per;
        if (q < cap && q >= n) continue;
        const int64_t src = q < cap ? static_cast<int64_t>(tok[q]) : q - cap;
        const uint4 w = reinterpret_cast<const uint4 *>(x + src * H)[v];
        uint4 o;
        o.x = __byte_perm(w.x, w.z, 0x5410);
        o.y = __byte_perm(w.x, w.z, 0x7632);
        o.z = __byte_perm(w.y, w.w, 0x5410);
        o.w = __byte_perm(w.y, w.w, 0x7632);
        reinterpret_cast<uint4 *>(xs + q * H)[v] = o;
    }
}

}  // namespace tc

int32_t tc_tile_tokens() { return tc::NT; }

bool tc_ok(int64_t H, int64_t I) {
    return H % tc::BM == 0 && I % tc::BM == 0 && H % tc::BK == 0 && I % tc::BK == 0 &&
           H <= (1 << 20) && I <= (1 << 20);
}

size_t tc_xs_bytes(int64_t T, int32_t k, int64_t H) {
    return static_cast<size_t>(T * k + T) * static_cast<size_t>(H) * sizeof(uint16_t);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        tried = true;
    }
    return fn;
}

// 2D map over a row-major [rows, cols] 16-bit matrix: box of 64 columns x 64
// rows, 128-byte swizzle (the K-major operand layout of the MMA).
static bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows <= 0) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {tc::BK, tc::BOX};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status run_tc_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k, int32_t E,
                        const moe_expert *experts, const moe_expert *shared, const int32_t *offsets,
                        const int32_t *tok, const int32_t *tile_off, const int32_t *list,
                        const float *w, void *h, void *xs, float *yp, unsigned *counters,
                        uint32_t *flags, cudaStream_t stream, cudaEvent_t ev_down) {
    using namespace tc;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    (void)counters;
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
    a.yp = yp;
    a.w = w;
    a.bits = 4;
    // expert-sorted copy of x (and the shared expert's copy) in the MMA's K
    // order, for the TMA loads of pass 1
    const int64_t t_sh = shared ? T : 0;
    uint16_t *xs16 = static_cast<uint16_t *>(xs);
    {
        const int64_t vecs = (T * k + t_sh) * (H / 8);
        int64_t grid = (vecs + 255) / 256;
        if (grid > 65535) grid = 65535;
        if (grid > 0) {
            gather_rows<<<static_cast<unsigned>(grid), 256, 0, stream>>>(x, tok, offsets + E, T * k, t_sh, H, xs16);
            if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
        }
    }
    TcMaps m1, m2;
    if (!make_map(&m1.b_main, xs16, T * k, H, true) ||
        !make_map(&m1.b_shared, xs16 + T * k * H, t_sh > 0 ? t_sh : T, H, true) ||
        !make_map(&m2.b_main, h, T * k + T, I, false))
        return MOE_ERR_CUDA;
    m2.b_shared = m2.b_main;
    {
        const size_t smem = Smem<2>::total;
        if (cudaFuncSetAttribute(tc_ffn<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        tc_ffn<1><<<sms, threads_of(1), smem, stream>>>(m1, a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (ev_down) record_stage_event(ev_down, stream);
    {
        const size_t smem = Smem<1>::total;
        if (cudaFuncSetAttribute(tc_ffn<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        tc_ffn<2><<<sms, threads_of(2), smem, stream>>>(m2, a);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace moe
