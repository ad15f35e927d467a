// rmsnorm.cu -- weightless RMSNorm rounded to bf16, the input of each MoE layer
// of a stack: out = bf16(v * r) with r = 1 / sqrt(mean(v^2) + eps), where r is
// formed in fp32 with IEEE square root and IEEE division (no fast-math) and the
// product is rounded to nearest-even bf16.
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) rmsnorm_bf16_kernel(const float *__restrict__ v, int64_t H,
                                                           float eps, uint16_t *__restrict__ out) {
    __shared__ float part[8];
    const int64_t t = blockIdx.x;
    const float *vr = v + t * H;
    float ss = 0.0f;
    for (int64_t j = threadIdx.x; j < H; j += blockDim.x) ss = fmaf(vr[j], vr[j], ss);
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); w++) tot += part[w];
    const float r = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
    uint16_t *orow = out + t * H;
    for (int64_t j = threadIdx.x; j < H; j += blockDim.x) {
        const __nv_bfloat16 b = __float2bfloat16_rn(vr[j] * r);
        orow[j] = *reinterpret_cast<const uint16_t *>(&b);
    }
}

moe_status launch_rmsnorm(const float *v, int64_t T, int64_t H, float eps, uint16_t *out,
                          cudaStream_t stream) {
    if (T == 0) return MOE_OK;
    rmsnorm_bf16_kernel<<<static_cast<unsigned>(T), 256, 0, stream>>>(v, H, eps, out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
