// decode.cu -- the routed-expert MoE layer for decode-size batches (T <= 8) as
// one persistent kernel.
//
// "Show HN: running GLM 5.2 on a slow computer", implemented features: a
// DeepSeek-V3 style sigmoid router (noaux_tc, routed_scaling_factor, shared
// expert), int4/int8/int2 experts with per-row scales decoded on use, and
// batch-union MoE (every unique expert of the batch read once).  Here every
// expert is resident in HBM and one launch does the whole layer:
//
//   router    the routed blocks compute G.x for their experts (exact bf16*fp32
//             products summed in fp64, rounded once), the sigmoid and the biased
//             score, and publish them; a counter tells every block when all
//             scores are out.  Each block then runs the group-limited top-k
//             of every token itself (all its consumer threads at once,
//             select_tokens) instead of waiting for one block to do it: no
//             serial tail between the router and the experts.
//   items     the (expert, token group) pairs of the batch: the shared expert's
//             token groups first, then every unique routed expert (ascending)
//             with its tokens in groups of TG.  A fixed set of blocks owns the
//             shared expert and starts streaming it at once, since it does not
//             depend on routing; the other blocks split the routed items' rows.
//   gate/up   rows of the items' gate and up matrices stream through a
//             shared-memory ring filled by bulk copies (one producer warp,
//             mbarrier hand-off); 18 consumer warps compute the dot products;
//             h = silu(s_g g) * (s_u u) is written per (token, slot) pair and a
//             per-item counter is raised.
//   down      the same ring streams the items' down rows; a block waits for its
//             item's counter before reading h; it writes per-pair outputs and
//             counts the finished rows of every 64-row tile of H; the block that
//             completes a tile adds the slots of each token in slot order, plus
//             the shared expert's row, and writes y (deterministic, no atomics
//             on y).
//
// Dot products are exact integer arithmetic: the activation slice of a warp
// (x in bf16, h in fp32) is scaled by a power of two 2^F chosen from its largest
// magnitude so that it becomes 23-bit signed integers X (exact for every value
// within 2^16 of that maximum, rounded to the nearest integer below it), split
// into three byte limbs; the unsigned weight codes c (int4/int2) or signed
// bytes (int8) meet the limbs in dp4a instructions with 32-bit integer
// accumulators, the code bias (8 for int4, 2 for int2) is folded into the
// accumulators' start values (-bias * sum X), and the limb sums of a warp are
// combined in fp64 (exact) before the row scale is applied and the result is
// rounded once to fp32.
#include <cstring>

#include "common.cuh"
#include "select.cuh"

namespace moe {
namespace dc {

constexpr int NCW = 18;                  // consumer warps
constexpr int THREADS = 32 * (NCW + 1);  // + one producer warp
constexpr int CTHREADS = 32 * NCW;
constexpr int STAGE_W = 36 * 1024;       // weight bytes per ring stage
constexpr int SC_SLOT = 512;             // row scales of one matrix per stage (16-byte aligned superset)
constexpr int STAGE = STAGE_W + 2 * SC_SLOT;
constexpr int NST = 4;                   // ring stages
constexpr int RSC_MAX = 1536;            // row scales of one sub-run (rows x matrices)
constexpr int ACT_BYTES = 24 * 1024;     // activation rows staged in shared memory (x or h)
constexpr int RDMAX = 4;                 // row-dots per consumer warp per stage
constexpr int MAXT = 8;
constexpr int MAXK = 32;
constexpr int MAXITEMS = 80;
constexpr int RED_BYTES = 24 * 1024;
constexpr int TILE = 64;
constexpr int RMAX_DN = 4096;            // rows per down sub-run
constexpr int MAXE = 256;

// Workspace header words (the header is zeroed by moe_workspace_init).
constexpr int HW_ROUTE = 16;   // router blocks that have published their scores
constexpr int HW_EXIT = 17;    // blocks that have finished
constexpr int HW_WAIT_US = kHdrWaitWord; // bound of every wait in microseconds (0: 2 s)
constexpr int HW_GU = 32;      // blocks that have finished every gate/up row
constexpr int HW_TILES = 256;  // [<= 768] down rows finished per 64-row tile of H

struct Item {
    int32_t expert;  // -1: the shared expert
    int32_t ntok;
    int32_t tok[2];
    int32_t hrow[2];  // row of h / yp: pair t*k+slot, or T*k+t for the shared expert
    int32_t ok_gu, ok_dn;  // the expert's matrices have this layer's shape (checked once)
    const uint8_t *gq, *uq, *dq;
    const float *gs, *us, *ds;
};

struct Args {
    const uint16_t *x;  // [T][H] bf16
    int32_t T, H, I;
    const float *G, *bias;
    int32_t E, k, n_group, topk_group;
    float rsf, topp;
    const moe_expert *experts;  // device [E]
    const moe_expert *shared;   // device, nullable
    float *y;                   // [T][H]
    int32_t accumulate;
    int32_t *idx_out;  // [T][k]
    float *w_out;      // [T][k]
    float *sb;         // [2][T][E]: scores, then biased scores
    float *h;          // [T*k + T][I]
    float *yp;         // [T*k + T][H]
    uint32_t *hdr;     // workspace header (flag word at 0)
    int32_t n_sblocks; // blocks that own the shared expert
};

// ---------------------------------------------------------------------------
// Per-width layout of one lane chunk (CH bytes of a row = CW 32-bit words).
// A word unpacks into NU registers of four byte-sized codes; byte i of unpack u
// of word w holds the code of column col(w, u, i).
// ---------------------------------------------------------------------------
template <int BITS>
struct Bt;
template <>
struct Bt<4> {  // nibbles: low = even column
    static constexpr int CH = 16, CW = 4, NU = 2, NCOL = 32, BIAS = 8, PARTS = 2;
    __device__ static __forceinline__ int col(int w, int u, int i) { return 8 * w + 2 * i + u; }
    __device__ static __forceinline__ uint32_t unpack(uint32_t v, int u) { return (v >> (4 * u)) & 0x0F0F0F0Fu; }
};
template <>
struct Bt<8> {  // two's-complement bytes
    static constexpr int CH = 16, CW = 4, NU = 1, NCOL = 16, BIAS = 0, PARTS = 4;
    __device__ static __forceinline__ int col(int w, int, int i) { return 4 * w + i; }
    __device__ static __forceinline__ uint32_t unpack(uint32_t v, int) { return v; }
};
template <>
struct Bt<2> {  // crumbs: lowest pair = lowest column
    static constexpr int CH = 8, CW = 2, NU = 4, NCOL = 32, BIAS = 2, PARTS = 2;
    __device__ static __forceinline__ int col(int w, int u, int i) { return 16 * w + 4 * i + u; }
    __device__ static __forceinline__ uint32_t unpack(uint32_t v, int u) { return (v >> (2 * u)) & 0x03030303u; }
};

// acc += sum_i code_i * limb_i over four bytes.  Codes are unsigned (int4,
// int2) or signed (int8); limbs 0 and 1 are unsigned bytes, limb 2 signed.
template <bool SIGNED_CODES, bool SIGNED_LIMB>
__device__ __forceinline__ int32_t dp4a(uint32_t codes, uint32_t limb, int32_t acc) {
    int32_t d;
    if constexpr (!SIGNED_CODES && !SIGNED_LIMB)
        asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(codes), "r"(limb), "r"(acc));
    else if constexpr (!SIGNED_CODES && SIGNED_LIMB)
        asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(codes), "r"(limb), "r"(acc));
    else if constexpr (SIGNED_CODES && !SIGNED_LIMB)
        asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(codes), "r"(limb), "r"(acc));
    else
        asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(codes), "r"(limb), "r"(acc));
    return d;
}

// The activation limbs of one token for one lane chunk: NL byte limbs of the
// integers X (the top one signed), laid out to meet the unpacked codes.
template <int BITS>
struct Limbs {
    uint32_t l[Bt<BITS>::CW][Bt<BITS>::NU][3];
    int32_t init[3];  // accumulator start values: -bias * sum of each limb
};

// Builds the NL limbs of a lane's NCOL activations v (zeros for an inactive
// lane) with the warp's shared exponent F: X = round(v * 2^F) with
// |X| < 2^(8 NL - 2), so every value within 2^(8 NL - 10) of the warp's largest
// magnitude is represented exactly (bf16 carries 8 significant bits) and smaller
// ones are rounded to the nearest integer.  The rounding uses the 1.5 * 2^23
// trick: v * 2^F is an exact power-of-two scaling and the fma's single rounding
// is round-to-nearest-even.  A slice whose largest magnitude is below 2^-106
// (or not finite) becomes zeros.  Returns F.
template <int BITS, int NL>
__device__ __forceinline__ int make_limbs(float (&v)[Bt<BITS>::NCOL], Limbs<BITS> &L) {
    using B = Bt<BITS>;
    constexpr int TOP = 8 * NL - 2;  // |X| < 2^TOP
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < B::NCOL; j++) m = fmaxf(m, fabsf(v[j]));
    m = warp_max(m);
    const int be = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu);
    const bool live = be >= TOP - 1 && be < 255;
    const int F = live ? TOP + 126 - be : 0;  // m < 2^(be - 126)
    const float scale = live ? __uint_as_float(static_cast<uint32_t>(F + 127) << 23) : 0.0f;
    const uint32_t ones = 0x01010101u;
    int32_t sx[3] = {0, 0, 0};
#pragma unroll
    for (int w = 0; w < B::CW; w++)
#pragma unroll
        for (int u = 0; u < B::NU; u++) {
            int32_t X[4];
#pragma unroll
            for (int i = 0; i < 4; i++)
                X[i] = __float_as_int(fmaf(v[B::col(w, u, i)], scale, 12582912.0f)) - 0x4B400000;
            const uint32_t ab = __byte_perm(X[0], X[1], 0x5140), cd = __byte_perm(X[2], X[3], 0x5140);
            L.l[w][u][0] = __byte_perm(ab, cd, 0x5410);  // byte 0 of each X
            L.l[w][u][1] = __byte_perm(ab, cd, 0x7632);  // byte 1
            sx[0] = dp4a<false, false>(L.l[w][u][0], ones, sx[0]);
            if constexpr (NL == 3) {
                const uint32_t ab2 = __byte_perm(X[0], X[1], 0x0062), cd2 = __byte_perm(X[2], X[3], 0x0062);
                L.l[w][u][2] = __byte_perm(ab2, cd2, 0x5410);  // byte 2 (signed)
                sx[1] = dp4a<false, false>(L.l[w][u][1], ones, sx[1]);
                sx[2] = dp4a<true, false>(L.l[w][u][2], ones, sx[2]);
            } else {
                L.l[w][u][2] = 0u;
                sx[1] = dp4a<true, false>(L.l[w][u][1], ones, sx[1]);  // byte 1 is the signed top limb
            }
        }
#pragma unroll
    for (int li = 0; li < 3; li++) L.init[li] = -B::BIAS * sx[li];
    return F;
}

// ---------------------------------------------------------------------------
// mbarrier, bulk copy, acquire/release helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bulk copy global -> shared, completion counted on the barrier; the weights
// are read once, so they are marked first in line for L2 eviction.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar, uint64_t pol) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
}
__device__ __forceinline__ void bulk_g2s_plain(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Named barrier of the consumer warps (the producer warp never joins it).
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(CTHREADS) : "memory"); }
struct ConsumerBar {
    static __device__ __forceinline__ void sync() { consumer_bar(); }
};
// Named barrier of consumers + producer (routed blocks, once routing is known).
__device__ __forceinline__ void block_bar2() { asm volatile("bar.sync 2, %0;" ::"n"(THREADS) : "memory"); }
// Barrier 3: the consumers signal (without waiting) that their router loads are
// issued; the producer waits for it before queueing its first copies, so that the
// gate rows are first in line.
__device__ __forceinline__ void loads_issued_arrive() { asm volatile("barrier.cta.arrive 3, %0;" ::"n"(THREADS) : "memory"); }
__device__ __forceinline__ void loads_issued_wait() { asm volatile("barrier.cta.sync 3, %0;" ::"n"(THREADS) : "memory"); }

struct Ctl {
    uint64_t limit_ns;
    volatile int *abort;
    uint32_t *flags;
};

__device__ __noinline__ void fail(uint32_t *flags, volatile int *abort) {
    raise_flag(flags, MOE_FLAG_WAIT_TIMEOUT);
    *abort = 1;
}

// Slow path of a bounded mbarrier wait (one thread); scalars only, so that the
// call keeps nothing in local memory.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t limit_ns, volatile int *abort,
                                            uint32_t *flags) {
    const uint64_t t0 = now_ns();
    while (true) {
        for (int i = 0; i < 64; i++)
            if (mbar_try(bar, parity)) return true;
        if (*abort) return false;
        if (now_ns() - t0 > limit_ns) {
            fail(flags, abort);
            return false;
        }
    }
}

// Bounded wait for an mbarrier phase (one thread).  Gives up at once when the
// block has aborted, or after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Ctl &c) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, c.limit_ns, c.abort, c.flags);
}

// Bounded wait until a global counter reaches target (one thread).
__device__ __noinline__ bool counter_wait_slow(const unsigned *p, unsigned target, uint64_t limit_ns,
                                               volatile int *abort, uint32_t *flags) {
    const uint64_t t0 = now_ns();
    while (true) {
        for (int i = 0; i < 16; i++) {
            if (ld_acquire(p) >= target) return true;
            __nanosleep(100);
        }
        if (*abort) return false;
        if (now_ns() - t0 > limit_ns) {
            fail(flags, abort);
            return false;
        }
    }
}
__device__ __forceinline__ bool counter_wait(const unsigned *p, unsigned target, const Ctl &c) {
    if (ld_acquire(p) >= target) return true;
    return counter_wait_slow(p, target, c.limit_ns, c.abort, c.flags);
}

// A matrix the ring can stream: this layer's shape, codes and scales 16-byte
// aligned (bulk copies need it).
__device__ __forceinline__ bool qmat_ok(const moe_qmat &m, int bits, int64_t rows, int64_t cols) {
    return m.q != nullptr && m.scale != nullptr && m.bits == bits && m.rows == rows && m.cols == cols &&
           (reinterpret_cast<uintptr_t>(m.q) & 15u) == 0 && (reinterpret_cast<uintptr_t>(m.scale) & 15u) == 0;
}

// Shared-memory layout of a block.
struct Smem {
    uint8_t ring[NST][STAGE];
    alignas(128) uint8_t act[ACT_BYTES];  // x rows (gate/up, router) or h rows (down) of the current tokens
    alignas(16) uint8_t red[RED_BYTES];  // dot-product partials; selection scratch before that
    float rsc[RSC_MAX];                  // row scales of the current sub-run [row][matrix]
    uint64_t full[NST], empty[NST];
    uint64_t actbar;  // completion of the staged activation / score copies
    Item items[MAXITEMS];
    int32_t sel_idx[MAXT * MAXK];
    float sel_w[MAXT * MAXK];
    int32_t prank[MAXT * MAXK];
    int32_t fexp[MAXT][NCW];  // exponent of the limbs of (token slot, k-slice warp)
    double lred[NCW][2][MAXT];
    int32_t my_tiles[768];
    int32_t tile_add[768];  // down rows this block finished per 64-row tile of H (counted once at the end)
    int32_t n_my_tiles;
    int32_t n_sitems, n_ritems;
    int32_t hstaged[MAXITEMS];  // byte offset of an item's h rows in act (-1: not staged)
    int abort;
};

// Consumer threads: copy n pieces (16-byte aligned sources, sizes multiples of
// 16) into shared memory at dst[i] with one bulk copy each, and wait for them.
// Every block reads the same few kilobytes of activations and scores; one bulk
// request per block keeps those L2 lines from being hit by thousands of small
// loads at once.  ph counts the uses of the barrier (the same in every
// consumer thread).
__device__ __forceinline__ void stage_copy(Smem &S, int n, const void *const *src, const uint32_t *bytes,
                                           uint8_t *const *dst, uint32_t &ph, const Ctl &c) {
    consumer_bar();  // nobody still reads the previous contents
    const uint32_t bar = smem_u32(&S.actbar);
    if (threadIdx.x == 0) {
        uint32_t tot = 0;
        for (int i = 0; i < n; i++) tot += bytes[i];
        mbar_expect(bar, tot);
        for (int i = 0; i < n; i++) bulk_g2s_plain(smem_u32(dst[i]), src[i], bytes[i], bar);
    }
    if ((threadIdx.x & 31) == 0 && !mbar_wait(bar, ph & 1u, c)) {
        // the block has aborted and uses the contents for nothing valid, but the
        // copies must land before the buffer is refilled or the block exits:
        // drain with the full two-second bound
        Ctl dr = c;
        dr.limit_ns = kFullWaitNs;
        volatile int never = 0;
        dr.abort = &never;
        mbar_wait(bar, ph & 1u, dr);
    }
    __syncwarp();
    ph++;
}

// Geometry of one phase (gate/up: M = 2 matrices of [I, H]; down: M = 1 of [H, I]).
struct Phase {
    int M;          // matrices per row
    int rowbytes;   // bytes per row of one matrix
    int chunks;     // lane chunks per row
    int KW, RG;     // k-slice warps, row groups
    int Rst;        // rows per stage
    int rmax;       // rows per sub-run
    int RI;         // rows per item
};

template <int BITS, int TG>
__device__ __forceinline__ Phase make_phase(int M, int64_t cols, int64_t RI, int rmax_cap) {
    using B = Bt<BITS>;
    Phase p;
    p.M = M;
    p.rowbytes = static_cast<int>(cols * BITS / 8);
    p.chunks = p.rowbytes / B::CH;
    p.KW = (p.chunks + 31) / 32;
    p.RG = NCW / p.KW;
    int r = STAGE_W / (M * p.rowbytes);
    const int r2 = RDMAX * p.RG / M;
    p.Rst = r < r2 ? r : r2;
    if (p.Rst < 1) p.Rst = 1;
    int rm = RED_BYTES / (M * TG * p.KW * 16);  // one entry: 4 int32 parts
    if (rm > rmax_cap) rm = rmax_cap;
    if (rm > 2 * CTHREADS / TG) rm = 2 * CTHREADS / TG;  // the epilogue: two rows per thread at most
    if (rm > RSC_MAX / M) rm = RSC_MAX / M;              // their scales
    p.rmax = rm;
    p.RI = static_cast<int>(RI);
    return p;
}

// ---------------------------------------------------------------------------
// Reduce-scatter butterfly: V values per lane in, lane keeps the warp sum of
// value bfly_idx<V>(lane) in v[0].
// ---------------------------------------------------------------------------
template <int V, int OFF>
struct IBfly {
    static __device__ __forceinline__ void run(int32_t *v, int lane) {
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < V / 2; i++) {
            const int32_t send = upper ? v[i] : v[i + V / 2];
            const int32_t keep = upper ? v[i + V / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
        }
        IBfly<V / 2, OFF / 2>::run(v, lane);
    }
};
template <int OFF>
struct IBfly<1, OFF> {
    static __device__ __forceinline__ void run(int32_t *v, int lane) {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
        IBfly<1, OFF / 2>::run(v, lane);
    }
};
template <>
struct IBfly<1, 0> {
    static __device__ __forceinline__ void run(int32_t *, int) {}
};
template <int V>
__device__ __forceinline__ int bfly_idx(int lane) {
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

// ---------------------------------------------------------------------------
// Phase sweeps.  The producer and the consumers walk the same plan: the block's
// rows [q0, q1) of its item class (rows of item m are [m*RI, (m+1)*RI)), in
// sub-runs that stay inside one item and hold at most rmax rows, each cut into
// stages of at most Rst rows.  The ring's stage counter st runs on across
// phases.
// ---------------------------------------------------------------------------
__device__ __forceinline__ const moe_expert *item_expert(const Args &a, const Item &it) {
    return it.expert < 0 ? a.shared : a.experts + it.expert;
}

// Fills the cached matrix pointers and shape checks of an item (one thread).
template <int BITS>
__device__ __forceinline__ void item_fill(const Args &a, Item &it) {
    const moe_expert *ex = item_expert(a, it);
    const moe_qmat g = ex->gate, u = ex->up, d = ex->down;
    it.ok_gu = qmat_ok(g, BITS, a.I, a.H) && qmat_ok(u, BITS, a.I, a.H);
    it.ok_dn = qmat_ok(d, BITS, a.H, a.I);
    if (!it.ok_gu || !it.ok_dn) raise_flag(a.hdr, MOE_FLAG_BAD_EXPERT_SHAPE);
    it.gq = g.q;
    it.uq = u.q;
    it.dq = d.q;
    it.gs = g.scale;
    it.us = u.scale;
    it.ds = d.scale;
}

template <int BITS>
__device__ void produce_phase(const Args &a, Smem &S, const Phase &P, int item_base, int64_t q0, int64_t q1,
                              bool down, uint32_t &st, uint32_t &issued_end, uint64_t pol, const Ctl &c) {
    // geometry and row pointers in registers: the copies below carry memory
    // clobbers, which would otherwise reload them from memory at every stage
    const int RI = P.RI, rmax = P.rmax, Rst = P.Rst, rowbytes = P.rowbytes, M = P.M;
    for (int64_t q = q0; q < q1;) {
        const int m = static_cast<int>(q / RI);
        const int r = static_cast<int>(q - static_cast<int64_t>(m) * RI);
        int nsub = RI - r;
        if (nsub > rmax) nsub = rmax;
        if (q1 - q < nsub) nsub = static_cast<int>(q1 - q);
        const Item &it = S.items[item_base + m];
        const bool ok = down ? it.ok_dn : it.ok_gu;
        const uint8_t *src0 = down ? it.dq : it.gq;
        const uint8_t *src1 = down ? nullptr : it.uq;
        const float *sc0 = down ? it.ds : it.gs;
        const float *sc1 = down ? nullptr : it.us;
        for (int u0 = 0; u0 < nsub; u0 += Rst) {
            const int n = nsub - u0 < Rst ? nsub - u0 : Rst;
            const int s = static_cast<int>(st % NST);
            bool go = !*c.abort;
            if (go && st >= NST) go = mbar_wait(smem_u32(&S.empty[s]), ((st / NST) - 1) & 1, c);
            // a consumer that gave up on a stage releases it with its copy possibly
            // still in flight, and only after it has set abort: look again, so that
            // no copy is ever queued into a buffer that may still be written
            if (go) go = !*c.abort;
            if (!go) {
                st++;
                continue;  // aborted: issue nothing more
            }
            const uint32_t bar = smem_u32(&S.full[s]);
            if (ok) {
                const uint32_t bytes = static_cast<uint32_t>(n) * rowbytes;
                // the rows' scales: the 16-byte aligned superset [row0 & ~3, (row0 + n + 3) & ~3)
                const int row0 = r + u0, sa = row0 & ~3, se = (row0 + n + 3) & ~3;
                const uint32_t sbytes = static_cast<uint32_t>(se - sa) * 4u;
                mbar_expect(bar, (bytes + sbytes) * M);
                const int64_t off = static_cast<int64_t>(row0) * rowbytes;
                bulk_g2s(smem_u32(S.ring[s]), src0 + off, bytes, bar, pol);
                bulk_g2s(smem_u32(S.ring[s] + STAGE_W), sc0 + sa, sbytes, bar, pol);
                if (!down) {
                    bulk_g2s(smem_u32(S.ring[s] + bytes), src1 + off, bytes, bar, pol);
                    bulk_g2s(smem_u32(S.ring[s] + STAGE_W + SC_SLOT), sc1 + sa, sbytes, bar, pol);
                }
            } else {
                mbar_arrive(bar);  // nothing to copy: complete the phase for the consumers
            }
            st++;
            issued_end = st;
        }
        q += nsub;
    }
}

// Builds the NL-limb activations of the item's tokens for this lane's chunk
// from the rows staged in S.act (x in bf16 for gate/up, h in fp32 for down):
// row (by_token ? tok[t] : t) of the staged block.  Records the exponents in
// S.fexp (one writer per k-slice).
template <int BITS, int TG, int NL>
__device__ __forceinline__ void load_item_limbs(const Args &a, Smem &S, const Item &it, bool down, bool by_token,
                                                int kw, int rg, int lane, int chunks, Limbs<BITS> (&L)[TG],
                                                int act_off) {
    using B = Bt<BITS>;
    const int chunk = kw * 32 + lane;
    const bool active = chunk < chunks;
    const int col0 = chunk * B::NCOL;
#pragma unroll
    for (int t = 0; t < TG; t++) {
        float v[B::NCOL];
        const bool have = active && t < it.ntok;
        const int row = by_token ? it.tok[t] : t;
        if (!down) {
            const uint16_t *src = reinterpret_cast<const uint16_t *>(S.act) + row * a.H + col0;
#pragma unroll
            for (int i = 0; i < B::NCOL / 8; i++) {
                uint4 q = make_uint4(0u, 0u, 0u, 0u);
                if (have) q = *reinterpret_cast<const uint4 *>(src + 8 * i);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    v[8 * i + 2 * j] = __uint_as_float(w4[j] << 16);
                    v[8 * i + 2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
                }
            }
        } else {
            const float *src = reinterpret_cast<const float *>(S.act + act_off) + row * a.I + col0;
#pragma unroll
            for (int i = 0; i < B::NCOL / 4; i++) {
                float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                if (have) q = *reinterpret_cast<const float4 *>(src + 4 * i);
                v[4 * i] = q.x;
                v[4 * i + 1] = q.y;
                v[4 * i + 2] = q.z;
                v[4 * i + 3] = q.w;
            }
        }
        const int F = make_limbs<BITS, NL>(v, L[t]);
        if (rg == 0 && lane == 0) S.fexp[t][kw] = F;
    }
}

// Partial sums a lane hands to the warp reduction per (row-dot, token): int4 /
// int2 combine the two low limbs as A1 * 256 + A0 (|.| < 2^30 over a warp) and
// keep the top one apart; int8 sums can reach 2^24 per limb, so each limb stays
// apart (padded to a power of two).
template <int BITS, int NL>
struct Parts {
    static constexpr int N = BITS == 8 ? (NL == 3 ? 4 : 2) : NL - 1;
};

// The row-dots of one stage for this warp (row-dot j = rg + i * RG, i < RDMAX,
// of the stage's n * M rows): all the chunk loads first, then the dp4a chains of
// every row-dot interleaved (RDMAX * TG * NL independent accumulators).
template <int BITS, int TG, int NL>
__device__ __forceinline__ void stage_dots(const uint8_t *stage, int nrd, int rowbytes, int chunk, bool lactive,
                                           int rg, int RG, const Limbs<BITS> (&L)[TG],
                                           int32_t (&v)[RDMAX * TG * Parts<BITS, NL>::N]) {
    using B = Bt<BITS>;
    constexpr bool SC = BITS == 8;
    uint32_t w[RDMAX][B::CW];
#pragma unroll
    for (int i = 0; i < RDMAX; i++) {
        const int j = rg + i * RG;
        if (lactive && j < nrd) {
            const uint8_t *p = stage + j * rowbytes + chunk * B::CH;
            if constexpr (B::CW == 4) {
                const uint4 q = *reinterpret_cast<const uint4 *>(p);
                w[i][0] = q.x; w[i][1] = q.y; w[i][2] = q.z; w[i][3] = q.w;
            } else {
                const uint2 q = *reinterpret_cast<const uint2 *>(p);
                w[i][0] = q.x; w[i][1] = q.y;
            }
        } else {
#pragma unroll
            for (int wi = 0; wi < B::CW; wi++) w[i][wi] = 0u;
        }
    }
    int32_t acc[RDMAX][TG][NL];
#pragma unroll
    for (int i = 0; i < RDMAX; i++)
#pragma unroll
        for (int t = 0; t < TG; t++)
#pragma unroll
            for (int li = 0; li < NL; li++) acc[i][t][li] = L[t].init[li];
#pragma unroll
    for (int wi = 0; wi < B::CW; wi++)
#pragma unroll
        for (int u = 0; u < B::NU; u++)
#pragma unroll
            for (int i = 0; i < RDMAX; i++) {
                const uint32_t codes = B::unpack(w[i][wi], u);
#pragma unroll
                for (int t = 0; t < TG; t++) {
                    acc[i][t][0] = dp4a<SC, false>(codes, L[t].l[wi][u][0], acc[i][t][0]);
                    if constexpr (NL == 3) {
                        acc[i][t][1] = dp4a<SC, false>(codes, L[t].l[wi][u][1], acc[i][t][1]);
                        acc[i][t][2] = dp4a<SC, true>(codes, L[t].l[wi][u][2], acc[i][t][2]);
                    } else {
                        acc[i][t][1] = dp4a<SC, true>(codes, L[t].l[wi][u][1], acc[i][t][1]);
                    }
                }
            }
    constexpr int P = Parts<BITS, NL>::N;
#pragma unroll
    for (int i = 0; i < RDMAX; i++)
#pragma unroll
        for (int t = 0; t < TG; t++) {
            int32_t *o = v + (i * TG + t) * P;
            if constexpr (BITS == 8) {
#pragma unroll
                for (int q = 0; q < P; q++) o[q] = q < NL ? acc[i][t][q < NL ? q : 0] : 0;
            } else {
                o[0] = acc[i][t][1] * 256 + acc[i][t][0];
                if constexpr (NL == 3) o[1] = acc[i][t][2];
            }
        }
}

// Epilogue of one sub-run (all consumer threads): rows [r, r + nsub) of item it;
// thread ctid handles entries e = ctid + j * CTHREADS (j < 2) of the sub-run's
// (row, token) pairs; the row scales came with the stages (S.rsc).  The warp sums of each row-dot are combined across k-slices in
// fp64 (exact), scaled by 2^-F and the row scale, and rounded once to fp32.
// Gate/up writes h = silu(g) * u; down writes the per-pair outputs.
template <int BITS, int TG>
__device__ __forceinline__ void sub_run_epilogue(const Args &a, Smem &S, const Item &it, bool down, int nl, int r,
                                                int nsub, int M, int KW) {
    const int ctid = threadIdx.x;
    const int32_t *red = reinterpret_cast<const int32_t *>(S.red);
    const bool ok = down ? it.ok_dn : it.ok_gu;
#pragma unroll
    for (int j = 0; j < 2; j++) {
        const int e = ctid + j * CTHREADS;
        if (e >= nsub * it.ntok) break;
        const int u = e / it.ntok, t = e - u * it.ntok;
        const int row = r + u;
        double d[2] = {0.0, 0.0};
        for (int mat = 0; mat < M; mat++) {
            for (int w = 0; w < KW; w++) {
                const int32_t *pp = red + (((u * M + mat) * TG + t) * KW + w) * 4;
                double dv;
                if (BITS == 8)
                    dv = (nl == 3 ? static_cast<double>(pp[2]) * 65536.0 : 0.0) + static_cast<double>(pp[1]) * 256.0 +
                         static_cast<double>(pp[0]);
                else
                    dv = (nl == 3 ? static_cast<double>(pp[1]) * 65536.0 : 0.0) + static_cast<double>(pp[0]);
                // times 2^-F, exact (F in [-114, 127])
                d[mat] += dv * __longlong_as_double(static_cast<long long>(1023 - S.fexp[t][w]) << 52);
            }
        }
        const float s0 = S.rsc[u * M], s1 = M > 1 ? S.rsc[u * M + 1] : 0.0f;
        if (!down) {
            float hv = 0.0f;
            if (ok) {
                const float g = static_cast<float>(d[0] * static_cast<double>(s0));
                const float uv = static_cast<float>(d[1] * static_cast<double>(s1));
                hv = silu(g) * uv;
            }
            a.h[static_cast<int64_t>(it.hrow[t]) * a.I + row] = hv;
        } else {
            const float yv = ok ? static_cast<float>(d[0] * static_cast<double>(s0)) : 0.0f;
            a.yp[static_cast<int64_t>(it.hrow[t]) * a.H + row] = yv;
        }
    }
}

// Completion accounting of the 64-row tiles of H, once per block after all its
// down rows (S.tile_add holds this block's rows per tile), and the combine of
// every tile this block completed: y[t][j] = (y) + sum over slots in slot order
// of w * yp[pair][j] + yp[shared t][j].  Consumer threads only.
__device__ __forceinline__ void tiles_and_combine(const Args &a, Smem &S, int n_items_total) {
    const int ctid = threadIdx.x;
    const int ntiles = a.H / TILE;
    if (ctid == 0) S.n_my_tiles = 0;
    __threadfence();  // this block's per-pair outputs before its counts
    consumer_bar();
    const int need = n_items_total * TILE;
    int32_t *tile_cnt = reinterpret_cast<int32_t *>(a.hdr + HW_TILES);
    for (int ct = ctid; ct < ntiles; ct += CTHREADS) {
        const int add = S.tile_add[ct];
        if (add > 0) {
            const int old = atomicAdd(tile_cnt + ct, add);
            if (old + add == need) S.my_tiles[atomicAdd(&S.n_my_tiles, 1)] = ct;
        }
    }
    consumer_bar();
    const int nt = S.n_my_tiles;
    if (nt > 0) __threadfence();
    const int T = a.T, k = a.k;
    for (int e = ctid; e < nt * TILE * T; e += CTHREADS) {
        const int ct = S.my_tiles[e / (TILE * T)];
        const int rem = e % (TILE * T);
        const int t = rem / TILE;
        const int64_t j = static_cast<int64_t>(ct) * TILE + rem % TILE;
        float acc = a.accumulate ? a.y[static_cast<int64_t>(t) * a.H + j] : 0.0f;
        for (int sl = 0; sl < k; sl++) {
            const int p = t * k + sl;
            if (S.sel_idx[p] >= 0) acc += S.sel_w[p] * __ldcg(a.yp + static_cast<int64_t>(p) * a.H + j);
        }
        if (a.shared) acc += __ldcg(a.yp + static_cast<int64_t>(T * k + t) * a.H + j);
        a.y[static_cast<int64_t>(t) * a.H + j] = acc;
    }
    for (int i = ctid; i < nt; i += CTHREADS) tile_cnt[S.my_tiles[i]] = 0;
}

__device__ __forceinline__ int token_sig(const Item &it) {
    return it.tok[0] | ((it.ntok > 1 ? it.tok[1] : 0) << 8) | (it.ntok << 16);
}

// Consumer side of one phase (gate/up: NL = 2 limbs of x; down: NL = 3 limbs of
// h): dot products into S.red stage by stage, then each sub-run's epilogue.
// L holds the current limbs and sig the tokens they belong to (gate/up items of
// the same tokens share them; -1: none).
template <int BITS, int TG, int NL>
__device__ __forceinline__ void run_phase(const Args &a, Smem &S, const Phase &P, bool DOWN, int item_base,
                                          int64_t q0, int64_t q1, uint32_t &st, const Ctl &c, int n_items_total,
                                          Limbs<BITS> (&L)[TG], int &sig, uint32_t &ph) {
    using B = Bt<BITS>;
    constexpr int PN = Parts<BITS, NL>::N;
    constexpr int V = RDMAX * TG * PN;
    const int ctid = threadIdx.x;
    const int warp = ctid >> 5, lane = ctid & 31;
    const int RI = P.RI, rmax = P.rmax, Rst = P.Rst, rowbytes = P.rowbytes, M = P.M, RG = P.RG, KW = P.KW;
    const int kw = warp % KW, rg = warp / KW;
    const bool wactive = rg < RG;
    const int chunk = kw * 32 + lane;
    const bool lactive = wactive && chunk < P.chunks;
    int32_t *red = reinterpret_cast<int32_t *>(S.red);
    int cur = -1;
    for (int64_t q = q0; q < q1;) {
        const int m = static_cast<int>(q / RI);
        const int r = static_cast<int>(q - static_cast<int64_t>(m) * RI);
        int nsub = RI - r;
        if (nsub > rmax) nsub = rmax;
        if (q1 - q < nsub) nsub = static_cast<int>(q1 - q);
        const int gm = item_base + m;
        const Item &it = S.items[gm];
        const bool ok = DOWN ? it.ok_dn : it.ok_gu;
        if (gm != cur) {
            const int want = DOWN ? -2 - gm : token_sig(it);
            if (want != sig) {
                // stage the item's activation rows (h rows for down; for gate/up
                // with more than two tokens, the x rows of its tokens -- with at
                // most two, every x row is staged already)
                const bool all_x = !DOWN && a.T <= 2;
                const int hoff = DOWN ? S.hstaged[gm] : -1;
                if (hoff >= 0) {
                    consumer_bar();
                } else if (!all_x) {
                    const void *src[2];
                    uint32_t bytes[2];
                    uint8_t *dst[2];
                    for (int t = 0; t < it.ntok; t++) {
                        if (DOWN) {
                            src[t] = a.h + static_cast<int64_t>(it.hrow[t]) * a.I;
                            bytes[t] = static_cast<uint32_t>(a.I) * 4u;
                        } else {
                            src[t] = a.x + static_cast<int64_t>(it.tok[t]) * a.H;
                            bytes[t] = static_cast<uint32_t>(a.H) * 2u;
                        }
                        dst[t] = S.act + t * bytes[0];
                    }
                    stage_copy(S, it.ntok, src, bytes, dst, ph, c);
                } else {
                    consumer_bar();
                }
                if (wactive)
                    load_item_limbs<BITS, TG, NL>(a, S, it, DOWN, all_x, kw, rg, lane, P.chunks, L, hoff >= 0 ? hoff : 0);
                sig = want;
            }
            cur = gm;
        }
        for (int u0 = 0; u0 < nsub; u0 += Rst) {
            const int n = nsub - u0 < Rst ? nsub - u0 : Rst;
            const int s = static_cast<int>(st % NST);
            bool go = true;
            if (lane == 0) go = mbar_wait(smem_u32(&S.full[s]), (st / NST) & 1, c);
            go = __shfl_sync(0xffffffffu, go ? 1 : 0, 0) != 0;
            if (go && ok && wactive) {
                int32_t v[V];
                stage_dots<BITS, TG, NL>(S.ring[s], n * M, rowbytes, chunk, lactive, rg, RG, L, v);
                IBfly<V, 16>::run(v, lane);
                if ((lane & (32 / V - 1)) == 0 || V >= 32) {
                    const int idx = bfly_idx<V>(lane);
                    const int part = idx % PN, t = (idx / PN) % TG, i = idx / (PN * TG);
                    const int j = rg + i * RG;
                    if (j < n * M && (BITS != 8 || part < NL)) {
                        const int mat = j >= n ? 1 : 0, u = j - mat * n;  // M <= 2
                        red[((((u0 + u) * M + mat) * TG + t) * KW + kw) * 4 + part] = v[0];
                        if (kw == 0 && part == 0 && t == 0)
                            S.rsc[(u0 + u) * M + mat] = reinterpret_cast<const float *>(
                                S.ring[s] + STAGE_W + mat * SC_SLOT)[u + ((r + u0) & 3)];
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&S.empty[s]));
            st++;
        }
        consumer_bar();
        sub_run_epilogue<BITS, TG>(a, S, it, DOWN, NL, r, nsub, M, KW);
        if (DOWN) {
            // this sub-run's rows per 64-row tile of H (one thread per tile)
            const int ta = r / TILE, tb = (r + nsub - 1) / TILE;
            for (int ct = ta + ctid; ct <= tb; ct += CTHREADS) {
                const int lo = ct * TILE > r ? ct * TILE : r;
                const int hi = (ct + 1) * TILE < r + nsub ? (ct + 1) * TILE : r + nsub;
                S.tile_add[ct] += hi - lo;
            }
        }
        consumer_bar();
        q += nsub;
    }
}

// ---------------------------------------------------------------------------
// Router phase (routed blocks): scores of experts rb, rb + NR, ... for all tokens.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double dot4d(float4 g, uint2 xv, double acc) {
    acc = fma(static_cast<double>(g.x), static_cast<double>(bf16_bits_to_float(xv.x & 0xffffu)), acc);
    acc = fma(static_cast<double>(g.y), static_cast<double>(bf16_bits_to_float(xv.x >> 16)), acc);
    acc = fma(static_cast<double>(g.z), static_cast<double>(bf16_bits_to_float(xv.y & 0xffffu)), acc);
    acc = fma(static_cast<double>(g.w), static_cast<double>(bf16_bits_to_float(xv.y >> 16)), acc);
    return acc;
}

__device__ __forceinline__ void router_scores(const Args &a, Smem &S, int rb, int NR, uint32_t &ph, const Ctl &c) {
    const int ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
    const int T = a.T, E = a.E;
    const int H4 = a.H / 4;
    bool arrived = false;
    const uint32_t xrow = static_cast<uint32_t>(a.H) * 2u;
    for (int e0 = rb; e0 < E; e0 += 2 * NR) {
        const int eA = e0, eB = e0 + NR;
        const bool hasB = eB < E;
        for (int c0 = 0; c0 < H4; c0 += CTHREADS * 4) {  // uniform trip count (barriers inside)
            float4 ga[4], gb[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const int cc = c0 + ctid + CTHREADS * i;
                const bool in = cc < H4;
                ga[i] = in ? __ldcs(reinterpret_cast<const float4 *>(a.G + static_cast<int64_t>(eA) * a.H) + cc)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
                gb[i] = (in && hasB) ? __ldcs(reinterpret_cast<const float4 *>(a.G + static_cast<int64_t>(eB) * a.H) + cc)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (!arrived) {
                loads_issued_arrive();
                arrived = true;
            }
            // x in groups of up to 2 tokens staged in shared memory (all of them
            // stay there for the gate/up phase when T <= 2)
            for (int t0 = 0; t0 < T; t0 += 2) {
                const int nt = T - t0 < 2 ? T - t0 : 2;
                if (T > 2 || (e0 == rb && c0 == 0)) {
                    const void *src[2] = {a.x + static_cast<int64_t>(t0) * a.H, a.x + static_cast<int64_t>(t0 + 1) * a.H};
                    const uint32_t bytes[2] = {xrow, xrow};
                    uint8_t *dst[2] = {S.act, S.act + xrow};
                    stage_copy(S, nt, src, bytes, dst, ph, c);
                }
                const uint16_t *xs = reinterpret_cast<const uint16_t *>(S.act);
                double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
#pragma unroll
                for (int tt = 0; tt < 2; tt++) {
                    if (tt >= nt) break;
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int cc = c0 + ctid + CTHREADS * i;
                        if (cc < H4) {
                            const uint2 xv = *reinterpret_cast<const uint2 *>(xs + tt * a.H + 4 * cc);
                            acc[0][tt] = dot4d(ga[i], xv, acc[0][tt]);
                            acc[1][tt] = dot4d(gb[i], xv, acc[1][tt]);
                        }
                    }
                }
#pragma unroll
                for (int tt = 0; tt < 2; tt++) {
                    if (tt >= nt) break;
                    const double va = warp_sum(acc[0][tt]);
                    const double vb = warp_sum(acc[1][tt]);
                    if (lane == 0) {
                        const int t = t0 + tt;
                        // partial over this chunk of H, accumulated per warp in a fixed order
                        S.lred[warp][0][t] = (c0 == 0 ? 0.0 : S.lred[warp][0][t]) + va;
                        S.lred[warp][1][t] = (c0 == 0 ? 0.0 : S.lred[warp][1][t]) + vb;
                    }
                }
            }
        }
        consumer_bar();
        if (ctid < 2 * T) {
            const int which = ctid / T, t = ctid % T;
            const int e = which ? eB : eA;
            if (which == 0 || hasB) {
                double v = 0.0;
                for (int w = 0; w < NCW; w++) v += S.lred[w][which][t];
                const float sc = sigmoid_score(static_cast<float>(v));
                a.sb[static_cast<int64_t>(t) * E + e] = sc;
                a.sb[static_cast<int64_t>(T) * E + static_cast<int64_t>(t) * E + e] = sc + a.bias[e];
            }
        }
        consumer_bar();
    }
    if (!arrived) loads_issued_arrive();
    if (T <= 2 && rb >= E) {  // no expert here: stage x all the same for the gate/up phase
        const void *src[2] = {a.x, a.x + a.H};
        const uint32_t bytes[2] = {xrow, xrow};
        uint8_t *dst[2] = {S.act, S.act + xrow};
        stage_copy(S, T, src, bytes, dst, ph, c);
    }
}

// Group-limited top-k of every token from the published scores, by all
// consumer threads at once (select_tokens), after one bulk copy of the scores
// into shared memory.
__device__ __forceinline__ void select_block(const Args &a, Smem &S, uint32_t &ph, const Ctl &c) {
    const int TE = a.T * a.E;
    float *s_all = reinterpret_cast<float *>(S.red);  // [T][E]
    float *b_all = s_all + TE;                          // [T][E]
    {
        const void *src[1] = {a.sb};
        const uint32_t bytes[1] = {static_cast<uint32_t>((2 * TE * 4 + 15) & ~15)};  // the region is padded to 256 B
        uint8_t *dst[1] = {S.red};
        stage_copy(S, 1, src, bytes, dst, ph, c);
    }
    select_tokens<ConsumerBar>(s_all, b_all, a.T, a.E, a.k, a.n_group, a.topk_group, a.rsf, a.topp, b_all + TE,
                               S.sel_idx, S.sel_w, threadIdx.x, CTHREADS);
}

// Selection of every token, then the routed items; consumer threads only.
template <int BITS>
__device__ __forceinline__ void select_and_items(const Args &a, Smem &S, int TG, uint32_t &ph, const Ctl &c) {
    const int ctid = threadIdx.x;
    const int T = a.T, E = a.E, k = a.k;
    select_block(a, S, ph, c);
    consumer_bar();
    // rank of each (token, slot) pair among the pairs of its expert, by token
    const int P = T * k;
    for (int p = ctid; p < P; p += CTHREADS) {
        const int e = S.sel_idx[p];
        int rank = -1;
        if (e >= 0 && e < E) {
            rank = 0;
            const int t = p / k;
            for (int qq = 0; qq < t * k; qq++) rank += S.sel_idx[qq] == e;
        }
        S.prank[p] = rank;
    }
    if (ctid == 0) S.n_ritems = 0;
    consumer_bar();
    const int ns = S.n_sitems;
    for (int p = ctid; p < P; p += CTHREADS) {
        const int rank = S.prank[p];
        if (rank < 0) continue;
        const int e = S.sel_idx[p];
        int base = 0, ne = 0;
        for (int qq = 0; qq < P; qq++) {
            const int eq = S.sel_idx[qq];
            if (S.prank[qq] >= 0 && eq < e && S.prank[qq] % TG == 0) base++;
            ne += S.prank[qq] >= 0 && eq == e;
        }
        Item &it = S.items[ns + base + rank / TG];
        const int slot = rank % TG;
        it.tok[slot] = p / k;
        it.hrow[slot] = p;
        if (slot == 0) {
            it.expert = e;
            it.ntok = ne - rank < TG ? ne - rank : TG;
            item_fill<BITS>(a, it);
            atomicAdd(&S.n_ritems, 1);
        }
    }
    consumer_bar();
}

// Every block owns 1/NB of the rows of four work lists, in this order: the
// shared expert's gate/up rows, the routed items' gate/up rows, the shared
// expert's down rows, the routed items' down rows.  The shared expert does not
// depend on routing, so its copies are issued at once and land while the router
// runs; down rows are copied ahead while the last gate/up rows are computed; a
// grid-wide count of finished blocks separates the gate/up and down phases (h
// is read only once every block has written its rows).
__device__ __forceinline__ void block_range(int64_t total, int b, int NB, int64_t &q0, int64_t &q1) {
    q0 = total * b / NB;
    q1 = total * (b + 1) / NB;
}

// Down phase: stage the h rows of every down item of this block (shared list,
// then routed list) with one bulk copy each and a single wait, when they fit in
// S.act; otherwise each item stages its own rows when the phase reaches it.
__device__ __forceinline__ void stage_block_h(const Args &a, Smem &S, const Phase &PD, int ns, int nr, uint32_t &ph,
                                              const Ctl &c) {
    const int b = blockIdx.x, NB = gridDim.x;
    const uint32_t rowb = static_cast<uint32_t>(a.I) * 4u;
    const void *src[8];
    uint32_t bytes[8];
    uint8_t *dst[8];
    int n = 0;
    uint32_t off = 0;
    bool fits = true;
    for (int i = threadIdx.x; i < MAXITEMS; i += CTHREADS) S.hstaged[i] = -1;
    consumer_bar();
    for (int list = 0; list < 2 && fits; list++) {
        const int cnt = list ? nr : ns, base = list ? ns : 0;
        int64_t q0, q1;
        block_range(static_cast<int64_t>(cnt) * PD.RI, b, NB, q0, q1);
        if (q1 <= q0) continue;
        for (int m = static_cast<int>(q0 / PD.RI); m <= static_cast<int>((q1 - 1) / PD.RI) && fits; m++) {
            const Item &it = S.items[base + m];
            if (n + it.ntok > 8 || off + it.ntok * rowb > static_cast<uint32_t>(ACT_BYTES)) {
                fits = false;
                break;
            }
            if (threadIdx.x == 0) S.hstaged[base + m] = static_cast<int>(off);
            for (int t = 0; t < it.ntok; t++) {
                src[n] = a.h + static_cast<int64_t>(it.hrow[t]) * a.I;
                bytes[n] = rowb;
                dst[n] = S.act + off;
                off += rowb;
                n++;
            }
        }
    }
    if (fits && n > 0) {
        stage_copy(S, n, src, bytes, dst, ph, c);
    } else {
        consumer_bar();
        for (int i = threadIdx.x; i < MAXITEMS; i += CTHREADS) S.hstaged[i] = -1;
    }
    consumer_bar();
}

// The consumer warps' whole part of the layer (router, selection, the four
// lists); one function, with the phase loop inlined once, so that the limbs stay
// in registers throughout.
template <int BITS, int TG>
__device__ __forceinline__ void consumer_main(const Args &a, Smem &S, const Phase &PG, const Phase &PD, const Ctl &c) {
    const int ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
    const int b = blockIdx.x, NB = gridDim.x, T = a.T;
    Limbs<BITS> L[TG];
    int sig = -1;
    uint32_t st = 0, ph = 0;
    router_scores(a, S, b, NB, ph, c);
    __threadfence();
    consumer_bar();
    if (ctid == 0) atomicAdd(reinterpret_cast<unsigned *>(a.hdr + HW_ROUTE), 1u);
    if (T == 1) {
        // every gate/up item of a single token reads token 0: build its limbs
        // while the other blocks finish their scores
        Item t0;
        t0.expert = -1;
        t0.ntok = 1;
        t0.tok[0] = t0.tok[1] = 0;
        const int kw = warp % PG.KW, rg = warp / PG.KW;
        if (rg < PG.RG) load_item_limbs<BITS, TG, 3>(a, S, t0, false, true, kw, rg, lane, PG.chunks, L, 0);
        sig = token_sig(t0);
    }
    for (int i = ctid; i < a.H / TILE; i += CTHREADS) S.tile_add[i] = 0;
    const int ns = S.n_sitems;
    int nall = ns;
    for (int list = 0; list < 4; list++) {
        const bool down = list >= 2, routed = (list & 1) != 0;
        if (list == 0) {
            if (ctid == 0)
                counter_wait(reinterpret_cast<const unsigned *>(a.hdr + HW_ROUTE), static_cast<unsigned>(NB), c);
            consumer_bar();
            select_and_items<BITS>(a, S, TG, ph, c);
            if (b == 0) {  // one block publishes the routing
                for (int p = ctid; p < T * a.k; p += CTHREADS) {
                    a.idx_out[p] = S.sel_idx[p];
                    a.w_out[p] = S.sel_w[p];
                }
            }
            block_bar2();  // the producer learns the routed items
            nall = ns + S.n_ritems;
        }
        if (list == 2) {
            // every block's h rows are written before any block reads h
            __threadfence();
            consumer_bar();
            if (ctid == 0) {
                atomicAdd(reinterpret_cast<unsigned *>(a.hdr + HW_GU), 1u);
                counter_wait(reinterpret_cast<const unsigned *>(a.hdr + HW_GU), static_cast<unsigned>(NB), c);
            }
            consumer_bar();
            stage_block_h(a, S, PD, ns, S.n_ritems, ph, c);
        }
        const Phase &P = down ? PD : PG;
        const int n = routed ? S.n_ritems : ns;
        int64_t q0, q1;
        block_range(static_cast<int64_t>(n) * P.RI, b, NB, q0, q1);
        run_phase<BITS, TG, 3>(a, S, P, down, routed ? ns : 0, q0, q1, st, c, nall, L, sig, ph);
    }
    tiles_and_combine(a, S, nall);
}

// Ring stages of the shared expert's gate/up rows of this block.
__device__ __forceinline__ int list0_stages(const Args &a, Smem &S, const Phase &PG) {
    int64_t q0, q1;
    block_range(static_cast<int64_t>(S.n_sitems) * PG.RI, blockIdx.x, gridDim.x, q0, q1);
    int n = 0;
    for (int64_t q = q0; q < q1;) {
        const int r = static_cast<int>(q % PG.RI);
        int nsub = PG.RI - r;
        if (nsub > PG.rmax) nsub = PG.rmax;
        if (q1 - q < nsub) nsub = static_cast<int>(q1 - q);
        n += (nsub + PG.Rst - 1) / PG.Rst;
        q += nsub;
    }
    return n;
}

// The producer lane's part: the same plan as the consumers, issuing the
// stages' bulk copies of lists [first, last].  st runs on across the calls;
// issued_end is the end of the stages actually issued (for the drain).
template <int BITS>
__device__ __noinline__ void producer_lists(const Args &a, Smem &S, const Phase &PG, const Phase &PD, const Ctl &c,
                                            int first, int last, uint32_t &st, uint32_t &issued_end) {
    const int b = blockIdx.x, NB = gridDim.x;
    const uint64_t pol = evict_first_policy();
    const int ns = S.n_sitems;
    for (int list = first; list <= last; list++) {
        const bool down = list >= 2, routed = (list & 1) != 0;
        if (list == 2) {
            // the down rows follow once every block has written its h rows, so
            // that the consumers' reads of h are not queued behind them
            counter_wait(reinterpret_cast<const unsigned *>(a.hdr + HW_GU), static_cast<unsigned>(NB), c);
        }
        const Phase &P = down ? PD : PG;
        const int n = routed ? S.n_ritems : ns;
        int64_t q0, q1;
        block_range(static_cast<int64_t>(n) * P.RI, b, NB, q0, q1);
        produce_phase<BITS>(a, S, P, routed ? ns : 0, q0, q1, down, st, issued_end, pol, c);
    }
}

template <int BITS, int TG>
__global__ void __launch_bounds__(THREADS, 1) decode_layer(Args a) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    Smem &S = *reinterpret_cast<Smem *>(dsm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NB = gridDim.x;
    const int T = a.T;
    const uint32_t wus = a.hdr[HW_WAIT_US];
    Ctl c;
    c.limit_ns = wus ? static_cast<uint64_t>(wus) * 1000ull : kFullWaitNs;
    c.abort = &S.abort;
    c.flags = a.hdr;

    if (tid == 0) {
        for (int s = 0; s < NST; s++) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), NCW);
        }
        mbar_init(smem_u32(&S.actbar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        S.abort = 0;
    }
    // shared-expert items: token groups of TG
    const int n_s = a.shared ? (T + TG - 1) / TG : 0;
    for (int i = tid; i < n_s; i += THREADS) {
        Item &it = S.items[i];
        it.expert = -1;
        it.ntok = T - i * TG < TG ? T - i * TG : TG;
        for (int s2 = 0; s2 < 2; s2++) {
            const int t = i * TG + s2;
            it.tok[s2] = t < T ? t : 0;
            it.hrow[s2] = a.k * T + (t < T ? t : 0);
        }
        item_fill<BITS>(a, it);
    }
    if (tid == 0) S.n_sitems = n_s;
    __syncthreads();

    const Phase PG = make_phase<BITS, TG>(2, a.H, a.I, 1 << 30);
    const Phase PD = make_phase<BITS, TG>(1, a.I, a.H, RMAX_DN);
    if (warp < NCW) {
        consumer_main<BITS, TG>(a, S, PG, PD, c);
    } else {
        uint32_t st = 0, issued_end = 0;
        loads_issued_wait();
        // the shared expert's gate/up stages go out before the routing is known
        // when they all fit in the ring (the consumers take them after selecting)
        const bool early = list0_stages(a, S, PG) <= NST;
        if (lane == 0 && early) producer_lists<BITS>(a, S, PG, PD, c, 0, 0, st, issued_end);
        __syncwarp();
        block_bar2();  // wait for the routing
        if (lane == 0) {
            producer_lists<BITS>(a, S, PG, PD, c, early ? 1 : 0, 3, st, issued_end);
            // drain: no bulk copy may still be writing this block's shared
            // memory when it exits (this wait keeps the full two-second bound)
            Ctl dr = c;
            dr.limit_ns = kFullWaitNs;
            volatile int never = 0;
            dr.abort = &never;
            const uint32_t first = issued_end > NST ? issued_end - NST : 0;
            for (uint32_t s2 = first; s2 < issued_end; s2++)
                mbar_wait(smem_u32(&S.full[s2 % NST]), (s2 / NST) & 1, dr);
        }
        __syncwarp();
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned done = atomicAdd(reinterpret_cast<unsigned *>(a.hdr + HW_EXIT), 1u);
        if (done == static_cast<unsigned>(NB) - 1) {
            // last block: every other block has finished with the counters
            a.hdr[HW_ROUTE] = 0;
            for (int i = 0; i < MAXITEMS; i++) a.hdr[HW_GU + i] = 0;
            if (*const_cast<volatile uint32_t *>(a.hdr) & MOE_FLAG_WAIT_TIMEOUT)
                for (int i = 0; i < a.H / TILE; i++) a.hdr[HW_TILES + i] = 0;
            __threadfence();
            a.hdr[HW_EXIT] = 0;
        }
    }
}

}  // namespace dc

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool fused_decode_ok(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg, int32_t bits) {
    if (T < 1 || T > dc::MAXT || H % 64 || I % 64) return false;
    if (cfg->n_experts > dc::MAXE || cfg->top_k > dc::MAXK) return false;
    if (T * cfg->top_k + T > dc::MAXITEMS) return false;  // items: routed pairs + shared groups
    if (H / dc::TILE > 768) return false;
    const int ch = bits == 2 ? 8 : 16;
    const int64_t kw_g = (H * bits / 8 / ch + 31) / 32, kw_d = (I * bits / 8 / ch + 31) / 32;
    if (kw_g > dc::NCW || kw_d > dc::NCW) return false;
    // one row of gate + up must fit a ring stage
    if (2 * H * bits / 8 > dc::STAGE || I * bits / 8 > dc::STAGE) return false;
    // selection scratch inside the partials buffer: scores and biased scores,
    // then the selection's own scratch
    const int64_t sel = static_cast<int64_t>(T) *
                        (2 * cfg->n_experts + select_scratch_words(cfg->n_experts, cfg->top_k, cfg->n_group, cfg->topk_group));
    if (sel * 4 > dc::RED_BYTES) return false;
    return true;
}

size_t fused_decode_smem() { return sizeof(dc::Smem) + 1024; }

template <int BITS, int TG>
static moe_status launch_fused(const dc::Args &a, cudaStream_t stream) {
    auto kern = dc::decode_layer<BITS, TG>;
    const size_t smem = sizeof(dc::Smem);
    static bool attr_set = false;  // per instantiation; setting it again is harmless
    if (!attr_set) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_set = true;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    dc::Args aa = a;
    aa.n_sblocks = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(dc::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // all blocks resident: they wait on one another
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, aa) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status run_fused_decode(const uint16_t *x, int64_t T, int64_t H, int64_t I, const float *gate,
                            const float *bias, const moe_router_cfg *cfg, int32_t bits,
                            const moe_expert *experts, const moe_expert *shared, float *y,
                            int32_t accumulate, int32_t *idx_out, float *w_out, float *sb, float *h,
                            float *yp, uint32_t *hdr, cudaStream_t stream) {
    dc::Args a;
    std::memset(&a, 0, sizeof(a));
    a.x = x;
    a.T = static_cast<int32_t>(T);
    a.H = static_cast<int32_t>(H);
    a.I = static_cast<int32_t>(I);
    a.G = gate;
    a.bias = bias;
    a.E = cfg->n_experts;
    a.k = cfg->top_k;
    a.n_group = cfg->n_group;
    a.topk_group = cfg->topk_group;
    a.rsf = cfg->routed_scaling_factor;
    a.topp = cfg->expert_topp;
    a.experts = experts;
    a.shared = shared;
    a.y = y;
    a.accumulate = accumulate;
    a.idx_out = idx_out;
    a.w_out = w_out;
    a.sb = sb;
    a.h = h;
    a.yp = yp;
    a.hdr = hdr;
    const bool tg1 = T == 1;
    switch (bits) {
    case 4: return tg1 ? launch_fused<4, 1>(a, stream) : launch_fused<4, 2>(a, stream);
    case 8: return tg1 ? launch_fused<8, 1>(a, stream) : launch_fused<8, 2>(a, stream);
    case 2: return tg1 ? launch_fused<2, 1>(a, stream) : launch_fused<2, 2>(a, stream);
    default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace moe
