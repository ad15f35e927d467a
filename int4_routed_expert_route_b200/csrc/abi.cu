// abi.cu -- the extern "C" entry points of include/moe.h: argument checks,
// workspace layout and the kernel sequence of each call.  Nothing here
// allocates device memory; all scratch lives in the caller's workspace.
#include <cstring>

#include "common.cuh"

namespace moe {

// Kernel launchers (one per translation unit).
moe_status launch_quantize(const float *, int64_t, int64_t, int32_t, uint8_t *, float *, cudaStream_t);
moe_status launch_route(const uint16_t *, int64_t, int64_t, const float *, const float *,
                        const moe_router_cfg *, int32_t *, float *, float *, double *, cudaStream_t);
size_t route_part_bytes(int64_t T, int64_t H, int E);
int route_ks_for(int64_t T, int64_t H);
moe_status launch_bucket(const int32_t *, int64_t, int32_t, int32_t, int32_t *, int32_t *, int32_t *,
                         int32_t *, int32_t *, int32_t *, int32_t *, uint32_t *, int32_t, int32_t *,
                         cudaStream_t);
struct GemvArgs;
moe_status launch_combine(float *, const float *, const int32_t *, const float *, int64_t, int64_t,
                          int32_t, bool, bool, cudaStream_t);
moe_status launch_rmsnorm(const float *, int64_t, int64_t, float, uint16_t *, cudaStream_t);
bool route_fused_ok(int64_t T, int64_t H);
moe_status launch_route_fused(const uint16_t *, int64_t, int64_t, const float *, const float *,
                              const moe_router_cfg *, int32_t *, float *, float *, unsigned *,
                              int32_t *, int32_t *, int32_t *, int32_t *, int32_t *, int32_t *,
                              int32_t *, uint32_t *, int32_t *, int32_t, cudaStream_t);
bool decode_ok(int64_t T, int64_t H, int64_t I, int32_t k, int32_t bits);
bool fused_decode_ok(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg, int32_t bits);
moe_status run_fused_decode(const uint16_t *x, int64_t T, int64_t H, int64_t I, const float *gate,
                            const float *bias, const moe_router_cfg *cfg, int32_t bits,
                            const moe_expert *experts, const moe_expert *shared, float *y,
                            int32_t accumulate, int32_t *idx_out, float *w_out, float *sb, float *h,
                            float *yp, uint32_t *hdr, cudaStream_t stream);
bool tc_ok(int64_t H, int64_t I);
int32_t tc_tile_tokens();
size_t tc_xs_bytes(int64_t T, int32_t k, int64_t H);
moe_status run_tc_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k, int32_t E,
                        const moe_expert *experts, const moe_expert *shared, const int32_t *offsets,
                        const int32_t *tok, const int32_t *tile_off, const int32_t *list,
                        const float *w, void *h, void *xs, float *yp, unsigned *counters,
                        uint32_t *flags, cudaStream_t stream, cudaEvent_t ev_down);
moe_status run_decode_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k,
                            int32_t bits, const moe_expert *experts, int32_t n_experts, const moe_expert *shared,
                            const int32_t *unique, const int32_t *n_unique, const int32_t *offsets,
                            const int32_t *tok, const int32_t *pos, const int32_t *idx,
                            const float *w, float *h, float *yp, int32_t *tile_cnt, float *y,
                            int32_t accumulate, uint32_t *flags, cudaStream_t stream,
                            cudaEvent_t ev_down);
moe_status run_gemv_layer(const uint16_t *x, int64_t T, int64_t H, int64_t I, int32_t k, int32_t bits,
                          const moe_expert *experts, const moe_expert *shared, const int32_t *unique,
                          const int32_t *n_unique, const int32_t *offsets, const int32_t *tok,
                          float *h, float *yp, uint32_t *flags, int64_t max_segments,
                          int64_t max_tok, cudaStream_t stream, cudaEvent_t ev_down);
moe_status run_gemv_single(const uint16_t *x, int64_t T, int64_t H, int64_t I, const moe_expert &e,
                           const int32_t *rows, const float *row_w, int64_t n_rows, float *h,
                           float *y, uint32_t *flags, cudaStream_t stream);

static constexpr size_t kAlign = 256;
// Workspace header of a layer call: flag word at 0, router ticket at 64, wait
// bound at 72 (kHdrWaitWord), tensor-path counters at 128, down
// tile-completion counters at 1024 (zeroed by moe_workspace_init).
static constexpr size_t kHeaderBytes = 4096;
static size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool cfg_ok(const moe_router_cfg *c) {
    if (!c) return false;
    const int E = c->n_experts, k = c->top_k, ng = c->n_group, tkg = c->topk_group;
    if (E < 1 || E > 1024 || k < 1 || k > 32 || ng < 1 || ng > 32 || tkg < 1) return false;
    if (E % ng || tkg > ng) return false;
    if (ng > 1 && E / ng < 2) return false;
    if (k > tkg * (E / ng)) return false;
    if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return false;
    if (!(c->expert_topp >= 0.0f)) return false;
    return true;
}

// Largest batch the CUDA-core path takes on; from kTensorMinT tokens on, AUTO
// picks the tensor-core grouped GEMM for int4 layers (measured: from about ten
// tokens on a batch selects dozens of experts, and the grouped GEMM streams them
// several times faster than the CUDA-core items kernels).
static constexpr int64_t kGemvMaxT = 4096;
static constexpr int64_t kTensorMinT = 9;

bool plan_layer(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg, int32_t path,
                LayerPlan *p) {
    if (!cfg_ok(cfg) || T < 0 || H <= 0 || I <= 0) return false;
    std::memset(p, 0, sizeof(*p));
    p->T = T;
    p->H = H;
    p->I = I;
    p->E = cfg->n_experts;
    p->k = cfg->top_k;
    p->path = path == MOE_PATH_AUTO ? (T >= kTensorMinT && tc_ok(H, I) ? MOE_PATH_TENSOR : MOE_PATH_GEMV)
                                    : path;
    p->route_ks = route_ks_for(T, H);
    const size_t P = static_cast<size_t>(T) * p->k;
    const size_t E = static_cast<size_t>(p->E);
    const size_t Pall = P + static_cast<size_t>(T);
    size_t o = 0;
    p->off_flags = o;   o = up(o + kHeaderBytes);
    p->off_part = o;    o = up(o + route_part_bytes(T, H, p->E));
    p->off_idx = o;     o = up(o + P * 4);
    p->off_w = o;       o = up(o + P * 4);
    p->off_counts = o;  o = up(o + E * 4);
    p->off_offsets = o; o = up(o + (E + 1) * 4);
    p->off_list = o;    o = up(o + P * 4);
    p->off_tok = o;     o = up(o + P * 4);
    p->off_pos = o;     o = up(o + P * 4);
    p->off_unique = o;  o = up(o + E * 4);
    p->off_nunique = o; o = up(o + 4);
    p->off_tiles = o;   o = up(o + (E + 2) * 4);
    p->off_h = o;       o = up(o + Pall * static_cast<size_t>(I) * 4);
    // per-pair down outputs; the tensor path first keeps its expert-sorted
    // copy of x here (read by pass 1, dead before pass 2 writes the partials)
    const size_t yp_bytes = Pall * static_cast<size_t>(H) * 4;
    const size_t xs_bytes = p->path == MOE_PATH_TENSOR ? tc_xs_bytes(T, p->k, H) : 0;
    p->off_yp = o;      o = up(o + (yp_bytes > xs_bytes ? yp_bytes : xs_bytes));
    p->total = o;
    return true;
}

}  // namespace moe

namespace moe {

// Per-stage timing events.  Inside a stream capture they must be recorded as
// external event nodes, or the graph keeps them as internal dependencies only.
void record_stage_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, s);
}

}  // namespace moe

namespace moe {
__global__ void set_header_word(uint32_t *word, uint32_t value) { *word = value; }
}  // namespace moe

using namespace moe;

#define CUDA_OK(x) ((x) == cudaSuccess)

extern "C" {

const char *moe_status_str(moe_status s) {
    switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_DEVICE_FLAG: return "MOE_ERR_DEVICE_FLAG";
    }
    return "MOE_STATUS_UNKNOWN";
}

int32_t moe_abi_version(void) { return 1; }

moe_status moe_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
    const size_t n = ws_bytes < kHeaderBytes ? ws_bytes : kHeaderBytes;
    return CUDA_OK(cudaMemsetAsync(ws, 0, n, stream)) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_workspace_status(const void *ws, cudaStream_t stream, uint32_t *flags_out) {
    if (!ws) return MOE_ERR_WORKSPACE;
    uint32_t f = 0;
    if (!CUDA_OK(cudaStreamSynchronize(stream))) return MOE_ERR_CUDA;
    if (!CUDA_OK(cudaMemcpy(&f, ws, sizeof(f), cudaMemcpyDeviceToHost))) return MOE_ERR_CUDA;
    if (flags_out) *flags_out = f;
    return f ? MOE_ERR_DEVICE_FLAG : MOE_OK;
}

moe_status moe_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint32_t wait_us, cudaStream_t stream) {
    if (!ws || ws_bytes < kHeaderBytes || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    uint32_t *word = static_cast<uint32_t *>(ws) + kHdrWaitWord;
    set_header_word<<<1, 1, 0, stream>>>(word, wait_us);
    return CUDA_OK(cudaGetLastError()) ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_quantize_rows(const float *w, int64_t rows, int64_t cols, int32_t bits,
                             uint8_t *q_out, float *scale_out, cudaStream_t stream) {
    if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
    if (bits != 2 && bits != 4 && bits != 8) return MOE_ERR_INVALID_ARG;
    if ((bits == 4 && cols % 2) || (bits == 2 && cols % 4)) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!w || !q_out || !scale_out)) return MOE_ERR_INVALID_ARG;
    return launch_quantize(w, rows, cols, bits, q_out, scale_out, stream);
}

size_t moe_route_workspace_bytes(int64_t T, int64_t H, const moe_router_cfg *cfg) {
    if (!cfg_ok(cfg) || T < 0 || H <= 0) return 0;
    return 256 + up(route_part_bytes(T, H, cfg->n_experts));
}

moe_status moe_route_topk(const uint16_t *x, int64_t T, int64_t H, const float *gate,
                          const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                          float *w_out, float *gap_out, void *ws, size_t ws_bytes,
                          cudaStream_t stream) {
    if (!cfg_ok(cfg) || T < 0 || H <= 0 || H % 64) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !gate || !bias || !idx_out || !w_out)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate)) return MOE_ERR_INVALID_ARG;
    const size_t need = moe_route_workspace_bytes(T, H, cfg);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    double *part = reinterpret_cast<double *>(static_cast<char *>(ws) + 256);
    return launch_route(x, T, H, gate, bias, cfg, idx_out, w_out, gap_out, part, stream);
}

moe_status moe_bucket(const int32_t *idx, int64_t T, int32_t k, int32_t E, int32_t *counts,
                      int32_t *offsets, int32_t *list, int32_t *unique, int32_t *n_unique,
                      cudaStream_t stream) {
    if (T < 0 || k < 1 || E < 1 || E > 1024 || T * k > (1ll << 24)) return MOE_ERR_INVALID_ARG;
    if ((T > 0 && !idx) || !counts || !offsets || !unique || !n_unique) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !list) return MOE_ERR_INVALID_ARG;
    return launch_bucket(idx, T, k, E, counts, offsets, list, nullptr, nullptr, unique, n_unique,
                         nullptr, 0, nullptr, stream);
}

static bool qmat_host_ok(const moe_qmat &m, int64_t rows, int64_t cols) {
    return m.q && m.scale && (m.bits == 2 || m.bits == 4 || m.bits == 8) && m.reserved == 0 &&
           m.rows == rows && m.cols == cols && aligned16(m.q);
}

size_t moe_expert_ffn_workspace_bytes(int64_t n_rows, int64_t H, int64_t I) {
    if (n_rows < 0 || H <= 0 || I <= 0) return 0;
    return 256 + up(static_cast<size_t>(n_rows) * static_cast<size_t>(I) * 4);
}

moe_status moe_expert_ffn(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                          const moe_expert *e, const int32_t *rows, const float *row_w,
                          int64_t n_rows, float *y, void *ws, size_t ws_bytes,
                          cudaStream_t stream) {
    if (T < 0 || H <= 0 || I <= 0 || H % 64 || I % 64 || !e) return MOE_ERR_INVALID_ARG;
    if (!rows) n_rows = T;
    if (n_rows < 0 || (rows == nullptr && n_rows != T)) return MOE_ERR_INVALID_ARG;
    if (n_rows > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    if (!qmat_host_ok(e->gate, I, H) || !qmat_host_ok(e->up, I, H) || !qmat_host_ok(e->down, H, I))
        return MOE_ERR_INVALID_ARG;
    if (e->gate.bits != e->up.bits || e->gate.bits != e->down.bits) return MOE_ERR_INVALID_ARG;
    const size_t need = moe_expert_ffn_workspace_bytes(n_rows, H, I);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (n_rows == 0) return MOE_OK;
    float *h = reinterpret_cast<float *>(static_cast<char *>(ws) + 256);
    return run_gemv_single(x, T, H, I, *e, rows, row_w, n_rows, h, y,
                           static_cast<uint32_t *>(ws), stream);
}

size_t moe_layer_workspace_bytes(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg) {
    LayerPlan p;
    if (!plan_layer(T, H, I, cfg, MOE_PATH_AUTO, &p)) return 0;
    return p.total;
}

size_t moe_layer_workspace_bytes_ex(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg,
                                    int32_t path) {
    if (path != MOE_PATH_AUTO && path != MOE_PATH_GEMV && path != MOE_PATH_TENSOR) return 0;
    LayerPlan p;
    if (!plan_layer(T, H, I, cfg, path, &p)) return 0;
    return p.total;
}

static void rec(cudaEvent_t *ev, int i, cudaStream_t s) {
    if (ev && ev[i]) record_stage_event(ev[i], s);
}

moe_status moe_layer_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                                const float *gate, const float *bias, const moe_router_cfg *cfg,
                                const moe_expert *experts, const moe_expert *shared,
                                int32_t weight_bits, float *y, int32_t *idx_out, float *w_out,
                                void *ws, size_t ws_bytes, int32_t path, int32_t accumulate,
                                cudaEvent_t *events, cudaStream_t stream) {
    if (!cfg_ok(cfg) || T < 0 || H <= 0 || I <= 0 || H % 64 || I % 64) return MOE_ERR_INVALID_ARG;
    if (weight_bits != 2 && weight_bits != 4 && weight_bits != 8) return MOE_ERR_INVALID_ARG;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_GEMV && path != MOE_PATH_TENSOR)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !gate || !bias || !experts || !y)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate) || !aligned16(y) || !aligned16(experts))
        return MOE_ERR_INVALID_ARG;
    LayerPlan p;
    // the tensor-core path takes int4 experts only: AUTO sends int8 / int2
    // layers to the CUDA-core path at every batch size (its workspace is no
    // larger than the one moe_layer_workspace_bytes sizes for AUTO)
    const int32_t eff_path = (path == MOE_PATH_AUTO && weight_bits != 4) ? MOE_PATH_GEMV : path;
    if (!plan_layer(T, H, I, cfg, eff_path, &p)) return MOE_ERR_INVALID_ARG;
    if (p.path == MOE_PATH_TENSOR && (!tc_ok(H, I) || weight_bits != 4)) return MOE_ERR_UNSUPPORTED;
    if (p.path == MOE_PATH_GEMV && T > kGemvMaxT) return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < p.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (T == 0) return MOE_OK;
    char *base = static_cast<char *>(ws);
    uint32_t *flags = reinterpret_cast<uint32_t *>(base + p.off_flags);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(base + p.off_idx);
    float *w = w_out ? w_out : reinterpret_cast<float *>(base + p.off_w);
    int32_t *counts = reinterpret_cast<int32_t *>(base + p.off_counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(base + p.off_offsets);
    int32_t *list = reinterpret_cast<int32_t *>(base + p.off_list);
    int32_t *tok = reinterpret_cast<int32_t *>(base + p.off_tok);
    int32_t *pos = reinterpret_cast<int32_t *>(base + p.off_pos);
    int32_t *unique = reinterpret_cast<int32_t *>(base + p.off_unique);
    int32_t *nunique = reinterpret_cast<int32_t *>(base + p.off_nunique);
    float *h = reinterpret_cast<float *>(base + p.off_h);
    float *yp = reinterpret_cast<float *>(base + p.off_yp);
    moe_status st;
    unsigned *counter = reinterpret_cast<unsigned *>(base + p.off_flags + 64);
    int32_t *tile_cnt = reinterpret_cast<int32_t *>(base + p.off_flags + 1024);
    float *logits = reinterpret_cast<float *>(base + p.off_part);

    if (p.path == MOE_PATH_GEMV && T >= 3 && fused_decode_ok(T, H, I, cfg, weight_bits)) {
        // 3..8 tokens: the whole layer in one persistent kernel whose blocks split
        // every expert's rows evenly (the kernels below give each expert a fixed
        // share of the blocks, which leaves most of them idle once a batch
        // selects dozens of experts; measured crossover between 2 and 3 tokens)
        rec(events, 0, stream);
        st = run_fused_decode(x, T, H, I, gate, bias, cfg, weight_bits, experts, shared, y, accumulate,
                              idx, w, logits, h, yp, flags, stream);
        if (st != MOE_OK) return st;
        for (int i = 1; i < 6; i++) rec(events, i, stream);
        return MOE_OK;
    }

    if (p.path == MOE_PATH_GEMV && route_fused_ok(T, H) && decode_ok(T, H, I, p.k, weight_bits)) {
        // decode-size batch: fused router + bucketing, then the two GEMV kernels
        rec(events, 0, stream);
        st = launch_route_fused(x, T, H, gate, bias, cfg, idx, w, logits, counter, counts, offsets,
                                list, tok, pos, unique, nunique, flags, tile_cnt,
                                static_cast<int32_t>(H / 64), stream);
        if (st != MOE_OK) return st;
        rec(events, 1, stream);
        rec(events, 2, stream);
        st = run_decode_layer(x, T, H, I, p.k, weight_bits, experts, cfg->n_experts, shared, unique, nunique,
                              offsets, tok, pos, idx, w, h, yp, tile_cnt, y, accumulate, flags,
                              stream, events ? events[3] : nullptr);
        if (st != MOE_OK) return st;
        rec(events, 4, stream);
        rec(events, 5, stream);
        return MOE_OK;
    }

    if (p.path == MOE_PATH_TENSOR) {
        int32_t *tile_off = reinterpret_cast<int32_t *>(base + p.off_tiles);
        unsigned *tc_counters = reinterpret_cast<unsigned *>(base + p.off_flags + 128);
        rec(events, 0, stream);
        st = launch_route(x, T, H, gate, bias, cfg, idx, w, nullptr,
                          reinterpret_cast<double *>(logits), stream);
        if (st != MOE_OK) return st;
        rec(events, 1, stream);
        st = launch_bucket(idx, T, p.k, p.E, counts, offsets, list, tok, pos, unique, nunique, flags,
                           tc_tile_tokens(), tile_off, stream);
        if (st != MOE_OK) return st;
        rec(events, 2, stream);
        st = run_tc_layer(x, T, H, I, p.k, p.E, experts, shared, offsets, tok, tile_off, list, w,
                          base + p.off_h, base + p.off_yp, yp, tc_counters, flags, stream,
                          events ? events[3] : nullptr);
        if (st != MOE_OK) return st;
        rec(events, 4, stream);
        st = launch_combine(y, yp, pos, w, T, H, p.k, shared != nullptr, accumulate != 0, stream);
        if (st != MOE_OK) return st;
        rec(events, 5, stream);
        return MOE_OK;
    }

    rec(events, 0, stream);
    st = launch_route(x, T, H, gate, bias, cfg, idx, w, nullptr,
                      reinterpret_cast<double *>(logits), stream);
    if (st != MOE_OK) return st;
    rec(events, 1, stream);
    st = launch_bucket(idx, T, p.k, p.E, counts, offsets, list, tok, pos, unique, nunique, flags, 0,
                       nullptr, stream);
    if (st != MOE_OK) return st;
    rec(events, 2, stream);
    const int64_t max_seg = (T * p.k < p.E ? T * p.k : p.E) + (shared ? 1 : 0);
    const int64_t max_tok = T;
    st = run_gemv_layer(x, T, H, I, p.k, weight_bits, experts, shared, unique, nunique, offsets, tok, h, yp,
                        flags, max_seg, max_tok, stream, events ? events[3] : nullptr);
    if (st != MOE_OK) return st;
    rec(events, 4, stream);
    st = launch_combine(y, yp, pos, w, T, H, p.k, shared != nullptr, accumulate != 0, stream);
    if (st != MOE_OK) return st;
    rec(events, 5, stream);
    return MOE_OK;
}

moe_status moe_layer_forward(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                             const float *gate, const float *bias, const moe_router_cfg *cfg,
                             const moe_expert *experts, const moe_expert *shared,
                             int32_t weight_bits, float *y, int32_t *idx_out, float *w_out,
                             void *ws, size_t ws_bytes, cudaStream_t stream) {
    return moe_layer_forward_ex(x, T, H, I, gate, bias, cfg, experts, shared, weight_bits, y,
                                idx_out, w_out, ws, ws_bytes, MOE_PATH_AUTO, 0, nullptr, stream);
}

moe_status moe_rmsnorm_bf16(const float *v, int64_t T, int64_t H, float eps, uint16_t *out,
                            cudaStream_t stream) {
    if (T < 0 || H <= 0 || (T > 0 && (!v || !out)) || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
    return launch_rmsnorm(v, T, H, eps, out, stream);
}

size_t moe_stack_workspace_bytes(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg) {
    const size_t l = moe_layer_workspace_bytes(T, H, I, cfg);
    if (!l) return 0;
    return l + up(static_cast<size_t>(T) * static_cast<size_t>(H) * 2);
}

moe_status moe_stack_forward(float *resid, int64_t T, int64_t H, int64_t I, int32_t n_layers,
                             const moe_layer_params *layers, const moe_router_cfg *cfg,
                             float eps, uint16_t *layer_inputs, int32_t *idx_out, void *ws,
                             size_t ws_bytes, cudaStream_t stream) {
    if (n_layers < 0 || (n_layers > 0 && !layers) || !cfg_ok(cfg)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !resid) return MOE_ERR_INVALID_ARG;
    const size_t lw = moe_layer_workspace_bytes(T, H, I, cfg);
    const size_t need = moe_stack_workspace_bytes(T, H, I, cfg);
    if (!lw || !ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (T == 0) return MOE_OK;
    uint16_t *xin_ws = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + lw);
    const int64_t k = cfg->top_k;
    for (int32_t l = 0; l < n_layers; l++) {
        uint16_t *xin = layer_inputs ? layer_inputs + static_cast<int64_t>(l) * T * H : xin_ws;
        moe_status st = launch_rmsnorm(resid, T, H, eps, xin, stream);
        if (st != MOE_OK) return st;
        st = moe_layer_forward_ex(xin, T, H, I, layers[l].gate, layers[l].bias, cfg,
                                  layers[l].experts, layers[l].shared, layers[l].weight_bits,
                                  resid,
                                  idx_out ? idx_out + static_cast<int64_t>(l) * T * k : nullptr,
                                  nullptr, ws, lw, MOE_PATH_AUTO, 1, nullptr, stream);
        if (st != MOE_OK) return st;
    }
    return MOE_OK;
}

}  // extern "C"
