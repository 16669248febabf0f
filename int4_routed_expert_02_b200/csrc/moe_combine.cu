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

constexpr int kCombineMaxThreads = 1024;  // one thread per 4 columns up to H = 4096
constexpr int kCombinePer = 2;            // groups of 4 columns per thread: H <= 8192

__global__ void __launch_bounds__(kCombineMaxThreads)
combine_kernel(const float *__restrict__ y, const float *__restrict__ sh, const float *__restrict__ wts, int H, int k,
               int with_shared, const uint16_t *__restrict__ h_in, float *__restrict__ m_out,
               uint16_t *__restrict__ h_out, int post_norm, float layer_scalar, float eps) {
    __shared__ float red[kCombineMaxThreads / 32];
    __shared__ float wk[kMaxK];
    const int t = blockIdx.x, H4 = H / 4;
    if (threadIdx.x < k) wk[threadIdx.x] = wts[(size_t)t * k + threadIdx.x];
    __syncthreads();
    const float4 *y4 = reinterpret_cast<const float4 *>(y) + (size_t)t * k * H4;
    float ss = 0.f;
    // four columns per thread and step, kept in registers for the second half;
    // the loads of 8 routed slots (and the shared row) are issued before any is
    // used; per column the sum runs over s = 0, 1, ... in order, then adds the
    // shared branch
    float4 mv[kCombinePer];
#pragma unroll
    for (int r = 0; r < kCombinePer; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
        mv[r] = m;
        if (i >= H4) continue;
        for (int s0 = 0; s0 < k; s0 += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = s0 + u < k ? __ldg(y4 + (size_t)(s0 + u) * H4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                // a zero weight adds nothing (0 * y = 0 for finite y); skipping it lets a
                // rank of an expert-parallel split leave the y rows of pairs it does not own unset
                if (s0 + u < k && wk[s0 + u] != 0.f) {
                    const float w = wk[s0 + u];
                    m.x = fmaf(w, v[u].x, m.x);
                    m.y = fmaf(w, v[u].y, m.y);
                    m.z = fmaf(w, v[u].z, m.z);
                    m.w = fmaf(w, v[u].w, m.w);
                }
            }
        }
        if (with_shared) {
            const float4 sv = __ldg(reinterpret_cast<const float4 *>(sh) + (size_t)t * H4 + i);
            m.x += sv.x;
            m.y += sv.y;
            m.z += sv.z;
            m.w += sv.w;
        }
        if (m_out) reinterpret_cast<float4 *>(m_out)[(size_t)t * H4 + i] = m;
        mv[r] = m;
        ss = fmaf(m.x, m.x, fmaf(m.y, m.y, fmaf(m.z, m.z, fmaf(m.w, m.w, ss))));
    }
    if (!h_out) return;
    ss = block_sum(ss, red);
    const float inv = post_norm ? 1.0f / sqrtf(ss / (float)H + eps) : 1.0f;
    // out = (h + m * inv) * layer_scalar for the thread's own columns, 4 at a time
#pragma unroll
    for (int r = 0; r < kCombinePer; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        if (i >= H4) continue;
        const uint2 hv = __ldg(reinterpret_cast<const uint2 *>(h_in + (size_t)t * H) + i);
        const float4 m = mv[r];
        const uint32_t o0 = f32_to_bf16_bits((bf16_bits_to_float(hv.x & 0xffffu) + m.x * inv) * layer_scalar);
        const uint32_t o1 = f32_to_bf16_bits((bf16_bits_to_float(hv.x >> 16) + m.y * inv) * layer_scalar);
        const uint32_t o2 = f32_to_bf16_bits((bf16_bits_to_float(hv.y & 0xffffu) + m.z * inv) * layer_scalar);
        const uint32_t o3 = f32_to_bf16_bits((bf16_bits_to_float(hv.y >> 16) + m.w * inv) * layer_scalar);
        reinterpret_cast<uint2 *>(h_out + (size_t)t * H)[i] = make_uint2(o0 | (o1 << 16), o2 | (o3 << 16));
    }
}

cudaError_t launch_combine(const float *y, const float *sh, const float *wts, int T, int H, int k, int with_shared,
                           const uint16_t *h_in, float *m_out, uint16_t *h_out, int post_norm, float layer_scalar,
                           float eps, cudaStream_t st) {
    const int threads = min(kCombineMaxThreads, ((H / 4 + 31) / 32) * 32);
    if ((long long)threads * kCombinePer < H / 4) return cudaErrorInvalidValue;
    combine_kernel<<<T, threads, 0, st>>>(y, sh, wts, H, k, with_shared, h_in, m_out, h_out, post_norm,
                                                     layer_scalar, eps);
    return cudaGetLastError();
}

// Expert-parallel selection (no counterpart in the pages, which run on one
// device): the pairs whose expert lies in [e_lo, e_hi) keep their gate
// weight, the others get 0; the active list keeps the experts in range.
__global__ void __launch_bounds__(256) ep_select_kernel(const int32_t *__restrict__ idx, const float *__restrict__ wts,
                                                        const int32_t *__restrict__ active, int n, int e_lo, int e_hi,
                                                        float *__restrict__ wts_out, int32_t *__restrict__ active_out) {
    for (int p = threadIdx.x; p < n; p += blockDim.x) {
        const int e = idx[p];
        wts_out[p] = (e >= e_lo && e < e_hi) ? wts[p] : 0.f;
    }
    if (threadIdx.x == 0) {
        const int na = active[0];
        int cnt = 0;
        for (int i = 0; i < na; ++i) {
            const int e = active[1 + i];
            if (e >= e_lo && e < e_hi) active_out[1 + cnt++] = e;
        }
        active_out[0] = cnt;
    }
}

cudaError_t launch_ep_select(const int32_t *idx, const float *wts, const int32_t *active, int n, int e_lo, int e_hi,
                             float *wts_out, int32_t *active_out, cudaStream_t st) {
    ep_select_kernel<<<1, 256, 0, st>>>(idx, wts, active, n, e_lo, e_hi, wts_out, active_out);
    return cudaGetLastError();
}

}  // namespace moe
