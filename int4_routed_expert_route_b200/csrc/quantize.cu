// quantize.cu -- per-row symmetric quantisation and packing (load time).
//
// Rule (the layer's stated int4 scheme; int8/int2 as in "Show HN: running GLM
// 5.2 on a slow computer", implemented features, and the ideipro.ru item):
//   m = max|w_row|, s = m / Qmax (IEEE fp32 division), q = clamp(roundf(w / s))
// with one IEEE fp32 division per element, halves away from zero, s = 0 and
// q = 0 for an all-zero row.  This file must be compiled without fast-math: the
// divisions and roundf decide integer codes and must round exactly as IEEE fp32.
#include "common.cuh"

namespace moe {

template <int BITS>
struct QSpec;
template <>
struct QSpec<4> {
    static constexpr float div = 7.0f;
    static constexpr int lo = -8, hi = 7, per_byte = 2, bias = 8;
};
template <>
struct QSpec<8> {
    static constexpr float div = 127.0f;
    static constexpr int lo = -128, hi = 127, per_byte = 1, bias = 0;
};
template <>
struct QSpec<2> {
    static constexpr float div = 1.5f;
    static constexpr int lo = -2, hi = 1, per_byte = 4, bias = 2;
};

template <int BITS>
__device__ __forceinline__ int code_of(float w, float s) {
    if (s == 0.0f) return 0;
    float v = __fdiv_rn(w, s);
    int q = static_cast<int>(roundf(v));
    q = q < QSpec<BITS>::lo ? QSpec<BITS>::lo : q;
    q = q > QSpec<BITS>::hi ? QSpec<BITS>::hi : q;
    return q;
}

// One warp per row: max-abs reduction, then each lane packs whole bytes.
template <int BITS>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const float *__restrict__ w,
                                                            int64_t rows, int64_t cols,
                                                            uint8_t *__restrict__ q_out,
                                                            float *__restrict__ scale_out) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const float *wr = w + row * cols;
    float m = 0.0f;
    for (int64_t j = lane; j < cols; j += 32) m = fmaxf(m, fabsf(wr[j]));
    m = warp_max(m);
    const float s = (m == 0.0f) ? 0.0f : __fdiv_rn(m, QSpec<BITS>::div);
    if (lane == 0) scale_out[row] = s;
    constexpr int PB = QSpec<BITS>::per_byte;
    const int64_t nbytes = (cols * BITS + 7) / 8;
    uint8_t *qr = q_out + row * nbytes;
    for (int64_t b = lane; b < nbytes; b += 32) {
        uint32_t byte = 0;
#pragma unroll
        for (int i = 0; i < PB; i++) {
            const int64_t j = b * PB + i;
            const int q = code_of<BITS>(wr[j], s);
            if (BITS == 8)
                byte = static_cast<uint8_t>(static_cast<int8_t>(q));
            else
                byte |= static_cast<uint32_t>(q + QSpec<BITS>::bias) << (i * BITS);
        }
        qr[b] = static_cast<uint8_t>(byte);
    }
}

moe_status launch_quantize(const float *w, int64_t rows, int64_t cols, int32_t bits,
                           uint8_t *q_out, float *scale_out, cudaStream_t stream) {
    if (rows == 0) return MOE_OK;
    const int warps = 8;
    const unsigned grid = static_cast<unsigned>((rows + warps - 1) / warps);
    switch (bits) {
    case 4: quantize_rows_kernel<4><<<grid, warps * 32, 0, stream>>>(w, rows, cols, q_out, scale_out); break;
    case 8: quantize_rows_kernel<8><<<grid, warps * 32, 0, stream>>>(w, rows, cols, q_out, scale_out); break;
    case 2: quantize_rows_kernel<2><<<grid, warps * 32, 0, stream>>>(w, rows, cols, q_out, scale_out); break;
    default: return MOE_ERR_INVALID_ARG;
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
