// common.cuh -- shared device helpers and the internal launch descriptors of
// the MoE layer library (sm_100a).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kWarp = 32;

// ----------------------------------------------------------------------------
// Device flag word (first 4 bytes of every workspace).
// ----------------------------------------------------------------------------
__device__ __forceinline__ void raise_flag(uint32_t *flags, uint32_t bit) {
    if (flags) atomicOr(flags, bit);
}

// Header word 18 (bytes 72..75 of a workspace): the bound, in microseconds, of
// every on-chip wait in the kernels that have any (0: two seconds).  Waits that
// drain copies or tensor-core work still in flight before a block exits keep the
// full two-second bound whatever it says.
constexpr int kHdrWaitWord = 18;
constexpr uint64_t kFullWaitNs = 2000000000ull;
__device__ __forceinline__ uint64_t wait_limit_ns(const uint32_t *hdr) {
    const uint32_t us = hdr ? *const_cast<const volatile uint32_t *>(hdr + kHdrWaitWord) : 0u;
    return us ? static_cast<uint64_t>(us) * 1000ull : kFullWaitNs;
}

// ----------------------------------------------------------------------------
// Small arithmetic helpers.
// ----------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan of one int per thread across the block; returns the prefix
// and writes the block total to *total (all threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const int nw = blockDim.x >> 5;
        int t = lane < nw ? warp_tot[lane] : 0;
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += n;
        }
        if (lane < nw) warp_tot[lane] = ti - t;  // exclusive warp offsets
        if (lane == 31) warp_tot[32] = ti;
    }
    __syncthreads();
    const int ex = warp_tot[wid] + inc - v;
    *total = warp_tot[32];
    __syncthreads();
    return ex;
}

// Packed pair of fp32 values in one 64-bit register (the sm_100 f32x2 datapath).
struct f2 {
    unsigned long long v;
};

__device__ __forceinline__ f2 f2_make(float lo, float hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ f2 f2_make_bits(uint32_t lo, uint32_t hi) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ float f2_lo(f2 a) { return __uint_as_float(static_cast<uint32_t>(a.v)); }
__device__ __forceinline__ float f2_hi(f2 a) { return __uint_as_float(static_cast<uint32_t>(a.v >> 32)); }
__device__ __forceinline__ float f2_sum(f2 a) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a.v));
    return lo + hi;
}

// acc += a * b  (two lanes, round-to-nearest, no contraction surprises)
__device__ __forceinline__ void f2_fma(f2 &acc, f2 a, f2 b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc.v) : "l"(a.v), "l"(b.v));
}
// a - b
__device__ __forceinline__ f2 f2_sub(f2 a, f2 b) {
    f2 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
    return r;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }
// SiLU with the hardware exponential and reciprocal (a few ulp of fp32): for h
// that is rounded to fp16 right after (relative 2^-11), where expf and an IEEE
// division only cost issue slots.
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// 128-bit streaming load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_stream8(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

// ----------------------------------------------------------------------------
// Workspace layout of one layer call (host computes, kernels receive pointers).
// ----------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before its predecessor ends; griddep_wait() blocks
// until the predecessor grid has completed and its writes are visible, and
// griddep_launch() lets the successor's blocks be scheduled early.  Both are
// no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

struct LayerPlan {
    int64_t T, H, I;
    int32_t E, k;
    int32_t path;      // MOE_PATH_GEMV or MOE_PATH_TENSOR
    int32_t route_ks;  // K-splits of the router logits
    size_t off_flags, off_part, off_idx, off_w, off_counts, off_offsets, off_list, off_tok,
        off_pos, off_unique, off_nunique, off_tiles, off_h, off_yp, total;
};

// Host: fills the plan for a layer call; returns false on an impossible size.
bool plan_layer(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg, int32_t path,
                LayerPlan *p);

}  // namespace moe
