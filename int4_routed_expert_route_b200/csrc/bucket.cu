// bucket.cu -- batch-union bucketing: a stable counting sort of the
// (token, slot) pairs of a batch by expert, so that each unique expert of the
// batch is streamed once and applied to all of its positions ("Show HN: running
// GLM 5.2 on a slow computer", implemented features, batch-union MoE).
//
// One 1024-thread block.  Warp w owns the contiguous pair range
// [w P / 32, (w + 1) P / 32) and counts its pairs per expert (ranks among equal
// experts of one 32-pair step come from __match_any_sync); one pass over the
// experts turns the 32 per-warp counts into exclusive prefixes in warp order
// and the experts' totals into offsets; each warp then walks its range again
// and places its pairs.  Pairs of earlier warps, earlier steps and lower lanes
// come first, which keeps the sort stable; there are four block barriers in
// all, independent of the batch size.
#include "common.cuh"

namespace moe {

constexpr int BK_THREADS = 1024;

struct BucketArgs {
    const int32_t *idx;
    int64_t P;  // T * k
    int32_t k, E;
    int32_t *counts, *offsets, *list, *tok, *pos, *unique, *n_unique;
    uint32_t *flags;
    int32_t ntile;      // tokens per N-chunk of the tensor-core path (0: no tile table)
    int32_t *tile_off;  // [E+1] exclusive prefix of ceil(count / ntile)
};

constexpr int BK_WARPS = BK_THREADS / 32;
constexpr int BK_BATCH = 8;  // 32-pair steps whose indices are loaded together

__global__ void __launch_bounds__(BK_THREADS) bucket_kernel(BucketArgs a) {
    extern __shared__ int sm[];
    const int E = a.E;
    int *wc = sm;                        // [32][E] per-warp counts, then per-warp cursors
    int *base = sm + BK_WARPS * E;       // [E] offsets
    int *wtot = sm + (BK_WARPS + 1) * E; // [33] scan scratch
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t r0 = a.P * wid / BK_WARPS, r1 = a.P * (wid + 1) / BK_WARPS;
    int *mine = wc + wid * E;

    for (int i = tid; i < BK_WARPS * E; i += BK_THREADS) wc[i] = 0;
    __syncthreads();
    // 1. per-warp counts over the warp's range
    bool bad = false;
    for (int64_t b0 = r0; b0 < r1; b0 += 32 * BK_BATCH) {
        int ev[BK_BATCH];
#pragma unroll
        for (int j = 0; j < BK_BATCH; j++) {
            const int64_t p = b0 + 32 * j + lane;
            ev[j] = p < r1 ? a.idx[p] : -1;
        }
#pragma unroll
        for (int j = 0; j < BK_BATCH; j++) {
            const int e = ev[j];
            if (e >= E) bad = true;
            const bool valid = e >= 0 && e < E;
            const unsigned m = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid && (__ffs(m) - 1) == lane) mine[e] += __popc(m);
            __syncwarp();
        }
    }
    if (__syncthreads_or(bad) && tid == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_INDEX);

    // 2. per expert (one per thread, E <= 1024): exclusive prefixes over the
    //    warps, then offsets, the unique list and the tile table
    {
        const int e = tid;
        int c = 0;
        if (e < E) {
            for (int w = 0; w < BK_WARPS; w++) {
                const int v = wc[w * E + e];
                wc[w * E + e] = c;
                c += v;
            }
        }
        int tot;
        const int off = block_exclusive_scan(c, wtot, &tot);
        const int nz = (c > 0) ? 1 : 0;
        int nu;
        const int upos = block_exclusive_scan(nz, wtot, &nu);
        int tiles = 0;
        if (a.ntile > 0) tiles = (c + a.ntile - 1) / a.ntile;
        int ntiles;
        const int toff = block_exclusive_scan(tiles, wtot, &ntiles);
        if (e < E) {
            a.counts[e] = c;
            a.offsets[e] = off;
            if (nz) a.unique[upos] = e;
            if (a.tile_off) a.tile_off[e] = toff;
            base[e] = off;
        }
        if (tid == 0) {
            a.offsets[E] = tot;
            *a.n_unique = nu;
            if (a.tile_off) a.tile_off[E] = ntiles;
        }
    }
    __syncthreads();

    // 3. each warp places its pairs, in pair order
    for (int64_t b0 = r0; b0 < r1; b0 += 32 * BK_BATCH) {
        int ev[BK_BATCH];
#pragma unroll
        for (int j = 0; j < BK_BATCH; j++) {
            const int64_t p = b0 + 32 * j + lane;
            ev[j] = p < r1 ? a.idx[p] : -1;
        }
#pragma unroll
        for (int j = 0; j < BK_BATCH; j++) {
            const int64_t p = b0 + 32 * j + lane;
            const int e = ev[j];
            const bool valid = e >= 0 && e < E;
            const unsigned m = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid) {
                const int q = base[e] + mine[e] + __popc(m & lanemask_lt());
                a.list[q] = static_cast<int32_t>(p);
                if (a.tok) a.tok[q] = static_cast<int32_t>(p / a.k);
                if (a.pos) a.pos[p] = q;
            } else if (p < r1 && a.pos) {
                a.pos[p] = -1;
            }
            __syncwarp();  // every lane has read the cursor before its leader moves it
            if (valid && (__ffs(m) - 1) == lane) mine[e] += __popc(m);
            __syncwarp();
        }
    }
}

size_t bucket_smem_bytes(int E) { return static_cast<size_t>((BK_WARPS + 1) * E + 40) * sizeof(int); }

moe_status launch_bucket(const int32_t *idx, int64_t T, int32_t k, int32_t E, int32_t *counts,
                         int32_t *offsets, int32_t *list, int32_t *tok, int32_t *pos,
                         int32_t *unique, int32_t *n_unique, uint32_t *flags, int32_t ntile,
                         int32_t *tile_off, cudaStream_t stream) {
    BucketArgs a;
    a.idx = idx;
    a.P = T * k;
    a.k = k;
    a.E = E;
    a.counts = counts;
    a.offsets = offsets;
    a.list = list;
    a.tok = tok;
    a.pos = pos;
    a.unique = unique;
    a.n_unique = n_unique;
    a.flags = flags;
    a.ntile = ntile;
    a.tile_off = tile_off;
    const size_t smem = bucket_smem_bytes(E);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    bucket_kernel<<<1, BK_THREADS, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
