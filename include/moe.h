/*
 * moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE layer library
 * (libmoe_b200.so).
 *
 * The layer (DeepSeek-V3 style sigmoid router with noaux_tc bias correction,
 * group-limited top-k, routed_scaling_factor and a shared expert, followed by
 * SwiGLU experts whose weights are int4/int8/int2 with one fp32 scale per row)
 * is the MoE block described in "Show HN: running GLM 5.2 on a slow computer"
 * (hi.news.hada.io), section "implemented features", and in "Enthusiast ran
 * GLM-5.2 on a laptop with 25 GB of RAM" (ideipro.ru): 8 of 256 experts per
 * token, ~19 MB per int4 expert, batch-union expert application.  Here every
 * expert is resident in device memory.
 *
 * Conventions for every entry point
 *  - Pointers are device pointers unless stated "host".  They belong to the
 *    caller; the library never allocates or frees device memory.  Scratch memory
 *    comes only from the caller's workspace `ws` (size from *_workspace_bytes).
 *  - Calls are asynchronous on `stream`: the host validates arguments, launches
 *    kernels and returns.  A host-side problem returns a status before anything
 *    is launched; a launch failure returns MOE_ERR_CUDA.  No exception crosses
 *    the ABI.
 *  - Problems only visible on the device (an out-of-range expert index in an
 *    input, an expert matrix whose shape does not match, an fp16 overflow of an
 *    intermediate) are latched as bits in a flag word at the start of `ws`; the
 *    kernels then skip the offending work.  moe_workspace_status() reads them.
 *  - bf16 tensors are passed as uint16_t bit patterns.  All tensors are dense
 *    row-major.  Device pointers must be 16-byte aligned.
 *  - The library keeps no global state; calls on different streams with
 *    different workspaces may run concurrently.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or configuration */
    MOE_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels implement */
    MOE_ERR_CUDA = 3,        /* a CUDA runtime call or a launch failed */
    MOE_ERR_WORKSPACE = 4,   /* ws is NULL or smaller than *_workspace_bytes */
    MOE_ERR_DEVICE_FLAG = 5  /* moe_workspace_status found a latched device flag */
} moe_status;

/* Bits of the device flag word (moe_workspace_status). */
#define MOE_FLAG_BAD_EXPERT_INDEX 0x1u /* routing index >= n_experts in an input */
#define MOE_FLAG_BAD_EXPERT_SHAPE 0x2u /* an expert matrix's bits/rows/cols disagree with H, I */
#define MOE_FLAG_FP16_OVERFLOW    0x4u /* |h| above the fp16 range on the tensor-core path */
#define MOE_FLAG_WAIT_TIMEOUT     0x8u /* a bounded on-chip wait gave up (results invalid) */

/*
 * One quantised matrix in the canonical packed layout (stated for the layer's
 * int4 weights: per-row scale, code stored as q+8, low nibble = even column):
 *   rows x cols codes, row-major, each row ceil(cols*bits/8) bytes, no padding.
 *   bits 4: byte m of a row = (q[2m]+8) | (q[2m+1]+8) << 4
 *   bits 2: byte m of a row = sum_{i<4} (q[4m+i]+2) << 2i   (q in [-2,1])
 *   bits 8: byte m of a row = (int8) q[m]
 *   scale[r] (fp32): the row's dequantised weights are q * scale[r].
 */
typedef struct moe_qmat {
    const uint8_t *q;
    const float *scale;
    int32_t bits;
    int32_t reserved; /* must be 0 */
    int64_t rows;
    int64_t cols;
} moe_qmat;

/* A SwiGLU expert: gate and up are [I, H], down is [H, I]; all three share bits. */
typedef struct moe_expert {
    moe_qmat gate, up, down;
} moe_expert;

/*
 * Router configuration ("Show HN", implemented features: sigmoid router,
 * noaux_tc, routed_scaling_factor).  n_experts experts in n_group contiguous
 * groups; a group's score is the sum of its two largest biased scores; the
 * topk_group best groups are kept; top_k experts are chosen from them.
 * expert_topp in (0,1) enables adaptive expert top-p (the "--topp" option of the
 * same page, under this library's reading: keep the smallest set of highest-
 * weight slots whose weights reach expert_topp * their sum, drop the others
 * with index -1 and weight 0, no renormalisation); 0 or >= 1 disables it.
 * Limits: n_experts <= 1024, n_group <= 32, top_k <= 32.
 */
typedef struct moe_router_cfg {
    int32_t n_experts;
    int32_t top_k;
    int32_t n_group;
    int32_t topk_group;
    float routed_scaling_factor;
    float expert_topp;
} moe_router_cfg;

/* ------------------------------------------------------------------------- */
/* Library plumbing below (status names, version, workspace header): the pages
 * have no counterpart; these exist because the library never allocates and
 * reports device-side problems through the caller's workspace. */

/* Human-readable status name (static storage). */
MOE_API const char *moe_status_str(moe_status s);

/* ABI version of this header (bumped on any signature change). */
MOE_API int32_t moe_abi_version(void);

/*
 * Clear the header of a workspace (its first 4 KiB, or ws_bytes if smaller:
 * the device flag word and the counters the layer kernels keep between calls),
 * async on stream.  Call once on a fresh workspace and after reading a latched
 * flag.
 */
MOE_API moe_status moe_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronise `stream`, read the device flag word of `ws` into *flags_out
 * (host, nullable) and return MOE_ERR_DEVICE_FLAG if any bit is set, else MOE_OK.
 * The flags stay latched until moe_workspace_init.
 */
MOE_API moe_status moe_workspace_status(const void *ws, cudaStream_t stream, uint32_t *flags_out);

/*
 * Bound every on-chip wait of the calls that use `ws` to wait_us microseconds
 * (0: the default of two seconds), async on stream.  The kernels that wait on
 * one another's progress inside a launch (the tensor-core passes, the fused
 * decode kernel) give up a wait after that long, latch MOE_FLAG_WAIT_TIMEOUT
 * and return with their results invalid; waits that drain copies or
 * tensor-core work already in flight keep the two-second bound.  The value is
 * stored in the workspace header, so moe_workspace_init resets it to the
 * default.  Errors: MOE_ERR_WORKSPACE if ws is NULL, misaligned or smaller
 * than 4 KiB; MOE_ERR_CUDA if the write cannot be queued.
 */
MOE_API moe_status moe_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint32_t wait_us, cudaStream_t stream);

/*
 * Per-row symmetric quantisation and packing (load time).
 * Source: "Show HN", implemented features (per-row scales, packed int4/int2,
 * int8); ideipro.ru item (packing checked bit for bit).  For each row r:
 *   m = max_j |w[r,j]|;  s = m / Qmax (fp32 IEEE division; Qmax = 7, 127, 1.5
 *   for bits 4, 8, 2);  q = clamp(roundf(w / s), qmin, qmax) with one fp32 IEEE
 *   division per element and halves rounded away from zero; a zero row gets
 *   s = 0 and q = 0.  Codes are packed in the moe_qmat layout.
 *   w        [rows, cols] fp32 (finite values)
 *   q_out    [rows, cols*bits/8] uint8
 *   scale_out[rows] fp32
 * cols must be even for bits 4 and a multiple of 4 for bits 2.
 */
MOE_API moe_status moe_quantize_rows(const float *w, int64_t rows, int64_t cols, int32_t bits,
                             uint8_t *q_out, float *scale_out, cudaStream_t stream);

/*
 * Router: sigmoid scores, noaux_tc bias-corrected group-limited top-k.
 * Source: "Show HN", implemented features (DeepSeek-V3 style sigmoid router,
 * noaux_tc, routed_scaling_factor).  Per token t:
 *   logit_e = G[e,:] . x_t  (exact products, accumulated in fp64, rounded to fp32)
 *   s_e = sigmoid(logit_e)  (evaluated in fp64, rounded to fp32)
 *   b_e = s_e + bias_e      (fp32; the bias steers the choice only)
 *   groups, candidates and top-k as in moe_router_cfg; idx in descending b,
 *   ties to the lower index; w_i = (s_{idx_i} / sum_i s_{idx_i}) * rsf in fp32.
 *   x      [T, H] bf16;  gate [E, H] fp32;  bias [E] fp32
 *   idx_out[T, k] int32;  w_out [T, k] fp32
 *   gap_out[T] fp32, nullable: min(b_(k) - best unchosen candidate b,
 *          last kept group score - best dropped group score); +inf if none.
 * ws: moe_route_workspace_bytes(T, H, cfg) bytes.
 */
MOE_API size_t moe_route_workspace_bytes(int64_t T, int64_t H, const moe_router_cfg *cfg);
MOE_API moe_status moe_route_topk(const uint16_t *x, int64_t T, int64_t H, const float *gate,
                          const float *bias, const moe_router_cfg *cfg, int32_t *idx_out,
                          float *w_out, float *gap_out, void *ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * moe_route_topk without a workspace, for callers that cannot allocate device
 * memory when they route (a fixed, pre-planned memory budget; code that must not
 * call an allocator because it may synchronise the device; a host that only holds
 * raw device pointers from another runtime).  The pages have no counterpart: this
 * is an interface convenience, with the same results as moe_route_topk.
 * Scratch comes from a 4 MiB array inside the library, present on every GPU that
 * loads the library until the process exits (moe_route_noalloc_max_scratch_bytes
 * returns its size).  A request whose scratch, moe_route_workspace_bytes(T, H, cfg)
 * minus 256, exceeds it returns MOE_ERR_WORKSPACE before anything is launched
 * (the scratch is T * n_experts fp32 logits: up to T = 4096 with 256 experts).
 * The first call on a device looks up the array's address (make it before any
 * stream capture); only a successful lookup is kept, so a call whose lookup
 * failed returns MOE_ERR_CUDA and the next call tries again.  All calls share
 * the array: calls that overlap on the GPU race and must be serialised by the
 * caller.  Allocates nothing.
 */
MOE_API size_t moe_route_noalloc_max_scratch_bytes(void);
MOE_API moe_status moe_route_topk_noalloc(const uint16_t *x, int64_t T, int64_t H,
                                          const float *gate, const float *bias,
                                          const moe_router_cfg *cfg, int32_t *idx_out,
                                          float *w_out, float *gap_out, cudaStream_t stream);

/*
 * Batch-union bucketing ("Show HN", implemented features: each unique expert
 * of a batch is read once and applied to every position routed to it).
 * A stable counting sort of the (token, slot) pairs p = t*k + slot by expert:
 *   idx     [T, k] int32 (entries < 0 are dropped pairs and are not listed)
 *   counts  [E] int32;  offsets [E+1] int32 (exclusive scan of counts)
 *   list    [T*k] int32: pairs of expert e at list[offsets[e] .. offsets[e+1]),
 *           in increasing p
 *   unique  [E] int32: experts with counts > 0, ascending; n_unique [1] int32
 * Needs T*k <= 2^24 and E <= 1024; no workspace (one launch of one block, its
 * counters in shared memory).
 * An index >= E latches nothing here (no ws): the call treats it as dropped;
 * moe_layer_forward checks indices itself.
 */
MOE_API moe_status moe_bucket(const int32_t *idx, int64_t T, int32_t k, int32_t E, int32_t *counts,
                      int32_t *offsets, int32_t *list, int32_t *unique, int32_t *n_unique,
                      cudaStream_t stream);

/*
 * One SwiGLU expert applied to a set of tokens, accumulated into y:
 *   y[t] += row_w * W_down( silu(W_gate x[t]) * (W_up x[t]) ),  W = q * scale,
 * fp32 accumulation.  Source: the layer's SwiGLU form y = W_down(silu(W_gate x)
 * * W_up x); "Show HN" (dequant-on-use, single rows kept in f32).
 *   x     [T, H] bf16
 *   e     HOST pointer to one moe_expert (its matrices are device memory)
 *   rows  [n_rows] int32 token indices, distinct, nullable (= 0..T-1, n_rows = T)
 *   row_w [n_rows] fp32, nullable (= 1)
 *   y     [T, H] fp32, accumulated (y[t] is read and written only for listed t)
 * ws: moe_expert_ffn_workspace_bytes(n_rows, H, I) bytes.
 */
MOE_API size_t moe_expert_ffn_workspace_bytes(int64_t n_rows, int64_t H, int64_t I);
MOE_API moe_status moe_expert_ffn(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                          const moe_expert *e, const int32_t *rows, const float *row_w,
                          int64_t n_rows, float *y, void *ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * The routed-expert MoE layer:
 *   y_t = sum_i w_{t,i} FFN_{idx_{t,i}}(x_t) + FFN_shared(x_t)
 * with the router of moe_route_topk, batch-union bucketing, and each unique
 * expert of the batch streamed once.  Source: "Show HN", implemented features
 * (router, shared expert, batch-union MoE).  The shared expert is unweighted.
 *   x       [T, H] bf16;  gate [E, H] fp32;  bias [E] fp32
 *   experts DEVICE array of E moe_expert;  shared DEVICE pointer, nullable
 *   weight_bits  4, 8 or 2: the bit width of every expert matrix (checked on the
 *           device; a mismatching expert latches MOE_FLAG_BAD_EXPERT_SHAPE)
 *   y       [T, H] fp32, overwritten
 *   idx_out [T, k] int32 and w_out [T, k] fp32, nullable (routing decision)
 * ws: moe_layer_workspace_bytes(T, H, I, cfg) bytes.
 * Paths (AUTO): one or two tokens run a fused router launch (logits, selection
 * and, for two tokens, bucketing; one token's k slots are its segments as they
 * are) and two streaming GEMV launches (int4 dot products as exact int32 dp4a
 * sums per lane chunk); 3..8 tokens run one persistent kernel (router,
 * selection, gate/up, down and combine, every expert's rows split evenly over
 * all SMs, exact integer dot products); from 9 tokens on, int4 layers run the
 * tcgen05 tensor-core grouped GEMM (int4 codes converted to bf16 / fp16 in
 * registers and written to tensor memory, fp32 accumulation in tensor memory,
 * h kept in fp16; H, I multiples of 128 only).  MOE_PATH_GEMV forces the
 * CUDA-core kernels.  AUTO runs int8 and int2 layers on the CUDA-core path at
 * every batch size (up to 4096 tokens).  Both paths write one
 * fp32 partial per (token, expert) pair and add the partials of a token in a
 * fixed order, so y is bitwise reproducible run to run on either path (the two
 * paths round differently from each other).
 */
#define MOE_PATH_AUTO 0
#define MOE_PATH_GEMV 1
#define MOE_PATH_TENSOR 2
MOE_API size_t moe_layer_workspace_bytes(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg);
/* Workspace of moe_layer_forward_ex for a forced path (AUTO as above). */
MOE_API size_t moe_layer_workspace_bytes_ex(int64_t T, int64_t H, int64_t I,
                                            const moe_router_cfg *cfg, int32_t path);
MOE_API moe_status moe_layer_forward(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                             const float *gate, const float *bias, const moe_router_cfg *cfg,
                             const moe_expert *experts, const moe_expert *shared,
                             int32_t weight_bits, float *y,
                             int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                             cudaStream_t stream);

/*
 * moe_layer_forward with two extra controls (same semantics otherwise):
 *   path    MOE_PATH_AUTO / MOE_PATH_GEMV / MOE_PATH_TENSOR
 *   events  HOST array of MOE_LAYER_EVENTS events, nullable: event i is recorded
 *           on `stream` before stage i (0 router, 1 bucket, 2 gate/up, 3 down,
 *           4 combine) and event 5 after the last stage, for per-stage timing.
 *           Null entries are skipped.  On the decode path the kernels overlap
 *           their start-up with their predecessor (programmatic dependent
 *           launch); an event recorded between two of them serialises them, so
 *           to time a whole call pass only events 0 and 5.  Inside a stream
 *           capture the events are recorded as external event nodes.
 *   accumulate  0: y is overwritten; 1: y += layer output (residual add).
 */
#define MOE_LAYER_EVENTS 6
MOE_API moe_status moe_layer_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I,
                                const float *gate, const float *bias, const moe_router_cfg *cfg,
                                const moe_expert *experts, const moe_expert *shared,
                                int32_t weight_bits, float *y,
                                int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                                int32_t path, int32_t accumulate, cudaEvent_t *events,
                                cudaStream_t stream);

/*
 * RMSNorm without weight, rounded to bf16 (the layer input of a stack):
 *   out[t,j] = bf16( v[t,j] * r[t] ),  r[t] = 1 / sqrt(mean_j v[t,j]^2 + eps),
 *   fp32 arithmetic with IEEE square root and division, nearest-even bf16.
 *   v [T, H] fp32;  out [T, H] bf16
 * Source: the pages run a token through 75 consecutive MoE layers ("Enthusiast
 * ran GLM-5.2 on a laptop with 25 GB of RAM"; "Show HN", "disk-streaming MoE
 * execution"); the norm between them is the model's pre-layer RMSNorm, taken
 * here without its learned weight (unit gamma) since no weights are loaded.
 * Errors: MOE_ERR_INVALID_ARG for T < 0, H <= 0, null pointers with T > 0, or
 * eps negative / NaN; no workspace.
 */
MOE_API moe_status moe_rmsnorm_bf16(const float *v, int64_t T, int64_t H, float eps, uint16_t *out,
                            cudaStream_t stream);

/*
 * A stack of MoE layers chained with residual adds and an RMSNorm before each
 * router (the decode of consecutive MoE layers of the model; 75 per token in
 * the pages):
 *   for l in 0..L-1:  xin = bf16(rmsnorm(resid));  resid += MoE_l(xin)
 *   resid        [T, H] fp32, in: x_0, out: x_L
 *   layers       HOST array of L moe_layer_params (device pointers inside)
 *   layer_inputs [L, T, H] bf16, nullable: each layer's xin
 *   idx_out      [L, T, k] int32, nullable
 * ws: moe_stack_workspace_bytes(T, H, I, cfg) bytes.
 */
typedef struct moe_layer_params {
    const float *gate;
    const float *bias;
    const moe_expert *experts; /* device array [E] */
    const moe_expert *shared;  /* device, nullable */
    int32_t weight_bits;       /* 4, 8 or 2 */
    int32_t reserved;          /* must be 0 */
} moe_layer_params;
MOE_API size_t moe_stack_workspace_bytes(int64_t T, int64_t H, int64_t I, const moe_router_cfg *cfg);
MOE_API moe_status moe_stack_forward(float *resid, int64_t T, int64_t H, int64_t I, int32_t n_layers,
                             const moe_layer_params *layers, const moe_router_cfg *cfg,
                             float eps, uint16_t *layer_inputs, int32_t *idx_out, void *ws,
                             size_t ws_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
