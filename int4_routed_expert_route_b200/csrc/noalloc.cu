// noalloc.cu -- moe_route_topk_noalloc: the router call for callers that cannot
// hand the library a workspace.
//
// Some callers cannot call cudaMalloc or obtain device memory at the point where
// they route tokens: code that runs under a fixed, pre-planned memory budget
// (an inference server that reserves every byte up front), code that must not
// call an allocator because the allocator may synchronise the device or take a
// global lock, or host code that only receives raw device pointers from another
// runtime.  For them this entry point takes its scratch (the router's partial
// logits) from a file-scope device array that lives in the library image.
//
// The array holds kRouteScratchBytes (4 MiB) on every GPU that loads the library,
// until the process exits.  Its device address is looked up with
// cudaGetSymbolAddress by the first call made while that device is current, and
// kept once the lookup succeeds; a failed lookup returns MOE_ERR_CUDA and is
// tried again by the next call.  That first call should happen before any stream
// capture.  All calls share
// the array, so calls whose kernels overlap on the GPU (different streams, or
// different host threads) race on it and must be serialised by the caller.  The
// router overwrites every scratch element it reads, so nothing needs clearing.
#include <mutex>

#include "common.cuh"

namespace moe {

moe_status launch_route(const uint16_t *, int64_t, int64_t, const float *, const float *,
                        const moe_router_cfg *, int32_t *, float *, float *, double *, cudaStream_t);
size_t route_part_bytes(int64_t T, int64_t H, int E);

constexpr size_t kRouteScratchBytes = static_cast<size_t>(4) << 20;

// Device-side scratch.  In host code this name is only a stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu[kMaxDevices];
static void *g_scratch_ptr[kMaxDevices];  // set once a lookup has succeeded

// Device address of the scratch array on the current device `dev`, looked up
// on first use; only a successful lookup is cached.
static void *scratch_address(int dev) {
    std::lock_guard<std::mutex> lock(g_scratch_mu[dev]);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) {
            cudaGetLastError();  // the failure is reported through the status, not left pending
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_route_noalloc_max_scratch_bytes(void) { return kRouteScratchBytes; }

extern "C" MOE_API moe_status moe_route_topk_noalloc(const uint16_t *x, int64_t T, int64_t H,
                                                     const float *gate, const float *bias,
                                                     const moe_router_cfg *cfg, int32_t *idx_out,
                                                     float *w_out, float *gap_out,
                                                     cudaStream_t stream) {
    // moe_route_workspace_bytes validates the configuration (0 = invalid).
    if (!cfg || T < 0 || H <= 0 || H % 64 || moe_route_workspace_bytes(T, H, cfg) == 0)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !gate || !bias || !idx_out || !w_out)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate)) return MOE_ERR_INVALID_ARG;
    if (route_part_bytes(T, H, cfg->n_experts) > kRouteScratchBytes) return MOE_ERR_WORKSPACE;
    if (T == 0) return MOE_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    void *scratch = scratch_address(dev);
    if (scratch == nullptr) return MOE_ERR_CUDA;
    return launch_route(x, T, H, gate, bias, cfg, idx_out, w_out, gap_out, static_cast<double *>(scratch),
                        stream);
}
