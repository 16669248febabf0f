// moe_combine.cu -- weighted combine of the routed branches and the shared
// branch, then normalisation, residual and layer scalar.
//
// TurboFieldfare introduction page (discuss.pytorch.kr), section
// "TurboFieldfare's expert streaming structure": the second command buffer
// sums the routed branches with the router weights, adds the shared branch,
// then applies normalisation, the residual and the layer scalar.  Reading:
//     m   = sum_s w[t,s] * y[t,s] + sh[t]
//     out = bf16((h + m / sqrt(mean(m^2) + eps)) * layer_scalar)   (post_norm)
//         = bf16((h + m) * layer_scalar)                            (otherwise)
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float *__restrict__ y, const float *__restrict__ sh, const float *__restrict__ wts, int H, int k,
               int with_shared, const uint16_t *__restrict__ h_in, float *__restrict__ m_out,
               uint16_t *__restrict__ h_out, int post_norm, float layer_scalar, float eps) {
    extern __shared__ float msh[];  // [H]
    __shared__ float red[kCombineThreads / 32];
    const int t = blockIdx.x;
    float wk[kMaxK];
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) wk[s] = s < k ? wts[(size_t)t * k + s] : 0.f;
    float ss = 0.f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        float m = 0.f;
#pragma unroll 8
        for (int s = 0; s < k; ++s) m = fmaf(wk[s], y[((size_t)t * k + s) * H + i], m);
        if (with_shared) m += sh[(size_t)t * H + i];
        if (m_out) m_out[(size_t)t * H + i] = m;
        msh[i] = m;
        ss = fmaf(m, m, ss);
    }
    if (!h_out) return;
    ss = block_sum(ss, red);
    const float inv = post_norm ? 1.0f / sqrtf(ss / (float)H + eps) : 1.0f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const float v = (bf16_bits_to_float(h_in[(size_t)t * H + i]) + msh[i] * inv) * layer_scalar;
        h_out[(size_t)t * H + i] = f32_to_bf16_bits(v);
    }
}

cudaError_t launch_combine(const float *y, const float *sh, const float *wts, int T, int H, int k, int with_shared,
                           const uint16_t *h_in, float *m_out, uint16_t *h_out, int post_norm, float layer_scalar,
                           float eps, cudaStream_t st) {
    const size_t smem = sizeof(float) * (size_t)H;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(combine_kernel), smem);
    if (e != cudaSuccess) return e;
    combine_kernel<<<T, kCombineThreads, smem, st>>>(y, sh, wts, H, k, with_shared, h_in, m_out, h_out, post_norm,
                                                     layer_scalar, eps);
    return cudaGetLastError();
}

}  // namespace moe
