// bucket.cu -- batch-union bucketing: a stable counting sort of the
// (token, slot) pairs of a batch by expert, so that each unique expert of the
// batch is streamed once and applied to all of its positions ("Show HN: running
// GLM 5.2 on a slow computer", implemented features, batch-union MoE).
//
// One 1024-thread block: a shared-memory histogram, a block scan, then the
// pairs in chunks of 1024 in pair order; inside a chunk the rank of a pair
// among equal experts comes from __match_any_sync within the warp plus a
// per-warp count table scanned across warps, which keeps the sort stable.
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

__global__ void __launch_bounds__(BK_THREADS) bucket_kernel(BucketArgs a) {
    extern __shared__ int sm[];
    const int E = a.E;
    int *cnt = sm;                    // [E] counts, then cursors
    int *ctot = sm + E;               // [E] chunk totals
    int *wtot = sm + 2 * E;           // [33] scan scratch
    uint16_t *wcnt = reinterpret_cast<uint16_t *>(sm + 2 * E + 40);  // [32][E]
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

    for (int e = tid; e < E; e += BK_THREADS) cnt[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int64_t p = tid; p < a.P; p += BK_THREADS) {
        const int e = a.idx[p];
        if (e >= E) bad = true;
        else if (e >= 0) atomicAdd(&cnt[e], 1);
    }
    if (__syncthreads_or(bad) && tid == 0) raise_flag(a.flags, MOE_FLAG_BAD_EXPERT_INDEX);

    // offsets, unique list, tile table (E <= 1024: one expert per thread)
    {
        const int e = tid;
        const int c = e < E ? cnt[e] : 0;
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
            cnt[e] = off;  // becomes the cursor
        }
        if (tid == 0) {
            a.offsets[E] = tot;
            *a.n_unique = nu;
            if (a.tile_off) a.tile_off[E] = ntiles;
        }
    }
    __syncthreads();

    for (int64_t base = 0; base < a.P; base += BK_THREADS) {
        for (int i = tid; i < 32 * E; i += BK_THREADS) wcnt[i] = 0;
        __syncthreads();
        const int64_t p = base + tid;
        const int e = (p < a.P) ? a.idx[p] : -1;
        const bool valid = (e >= 0 && e < E);
        const int key = valid ? e : -1;
        const unsigned mask = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(mask & lanemask_lt());
        const bool leader = (__ffs(mask) - 1) == lane;
        if (valid && leader) wcnt[wid * E + e] = static_cast<uint16_t>(__popc(mask));
        __syncthreads();
        for (int ee = tid; ee < E; ee += BK_THREADS) {
            int run = 0;
            for (int w = 0; w < 32; w++) {
                const int c = wcnt[w * E + ee];
                wcnt[w * E + ee] = static_cast<uint16_t>(run);
                run += c;
            }
            ctot[ee] = run;
        }
        __syncthreads();
        if (valid) {
            const int q = cnt[e] + wcnt[wid * E + e] + rank;
            a.list[q] = static_cast<int32_t>(p);
            if (a.tok) a.tok[q] = static_cast<int32_t>(p / a.k);
            if (a.pos) a.pos[p] = q;
        } else if (p < a.P && a.pos) {
            a.pos[p] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += BK_THREADS) cnt[ee] += ctot[ee];
        __syncthreads();
    }
}

size_t bucket_smem_bytes(int E) {
    return static_cast<size_t>(2 * E + 40) * sizeof(int) + static_cast<size_t>(32) * E * sizeof(uint16_t);
}

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
