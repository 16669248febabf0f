// moe_router.cu -- the router of the MoE layer.
//
// TurboFieldfare introduction page (discuss.pytorch.kr), section
// "TurboFieldfare's expert streaming structure", router pseudo-code:
//   router_input = rmsnorm_no_scale(hidden)
//   scaled_input = router_input * router_scale / sqrt(hidden_size)
//   logits       = int8_affine(scaled_input)       (8-bit MLX affine, groups of 64)
//   topk         = highest_k(logits)
//   weights      = softmax(logits[topk]) * per_expert_scale[topk]
// The norm, the scaling and the projection accumulate in fp64 so the top-k
// decision does not depend on summation order; the experts' input
// xe = bf16(router_input) is written on the way.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kRouterThreads = 256;                   // 8 warps, each `epw` experts
constexpr int kRouterRows = kRouterThreads / kWarp;

// Dynamic shared memory: xsT[16][ld] (xs transposed so that lane c of a warp
// reading code m of its 16-byte chunk c hits consecutive doubles; ld = H/16
// rounded up to odd so that the transposing writes spread over the banks),
// csum[H/16] (sum of xs over each 16-column chunk), red[8].
__global__ void __launch_bounds__(kRouterThreads)
router_logits_kernel(const uint32_t *__restrict__ rq, const uint16_t *__restrict__ rs,
                     const uint16_t *__restrict__ rb, const uint16_t *__restrict__ router_scale,
                     const uint16_t *__restrict__ h, int H, int E, int epw, float eps, double *__restrict__ logits,
                     uint16_t *__restrict__ xe) {
    extern __shared__ double smem_d[];
    const int nchunk = H / 16;
    const int ld = nchunk | 1;
    double *xsT = smem_d;
    double *csum = xsT + (size_t)16 * ld;
    double *red = csum + nchunk;
    const int t = blockIdx.y;
    const uint16_t *ht = h + (size_t)t * H;

    // rmsnorm_no_scale in fp64
    double ss = 0.0;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const double v = (double)bf16_bits_to_float(ht[i]);
        ss += v * v;
    }
    ss = block_sum(ss, red);
    // one division per CTA: x / r is taken as x * (1 / r), which differs from
    // the quotient by at most an ulp of fp64 -- far below what moves a logit
    // gap or a BF16 rounding
    const double rinv = 1.0 / sqrt(ss / (double)H + (double)eps);
    const double inv_sqrt_h = 1.0 / sqrt((double)H);
    const bool write_xe = (xe != nullptr) && blockIdx.x == 0;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const double xn = (double)bf16_bits_to_float(ht[i]) * rinv;
        const double xs = xn * (double)bf16_bits_to_float(router_scale[i]) * inv_sqrt_h;
        xsT[(i & 15) * ld + (i >> 4)] = xs;
        if (write_xe) xe[(size_t)t * H + i] = f64_to_bf16_bits(xn);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
        double s = 0.0;
#pragma unroll
        for (int m = 0; m < 16; ++m) s += xsT[m * ld + c];
        csum[c] = s;
    }
    __syncthreads();

    // warp w takes experts blockIdx.x * 8 * epw + j * 8 + w, j < epw (the
    // norm above is shared by all of them)
    const int lane = threadIdx.x & 31;
    const int G = H / kGroup;
    for (int j = 0; j < epw; ++j) {
        const int e = (blockIdx.x * epw + j) * kRouterRows + (threadIdx.x >> 5);
        if (e >= E) break;
        const uint32_t *row = rq + (size_t)e * (H / 4);
        double acc = 0.0;
        for (int c = lane; c < nchunk; c += kWarp) {
            const uint4 q = ldg_nc_v4(row + 4 * c);
            const int g = c >> 2;  // four 16-code chunks per group of 64
            const double s = (double)bf16_bits_to_float(rs[(size_t)e * G + g]);
            const double b = (double)bf16_bits_to_float(rb[(size_t)e * G + g]);
            const uint32_t words[4] = {q.x, q.y, q.z, q.w};
            double dot = 0.0;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                for (int bi = 0; bi < 4; ++bi) {
                    const int m = wi * 4 + bi;
                    // the 8-bit code as a double: 2^52 + q read as fp64, minus 2^52 (exact,
                    // and an add instead of an integer-to-double conversion)
                    const double qd =
                        __hiloint2double(0x43300000, (int)((words[wi] >> (8 * bi)) & 0xffu)) - 4503599627370496.0;
                    dot += qd * xsT[m * ld + c];
                }
            }
            acc += s * dot + b * csum[c];
        }
        acc = warp_sum(acc);
        if (lane == 0) logits[(size_t)t * E + e] = acc;
    }
}

// One warp per token.  k rounds of a warp-wide argmax over the logits not yet
// taken, ordered by (logit desc, index asc), then the softmax over the k
// selected logits in fp64, times per_expert_scale.
__global__ void __launch_bounds__(kWarp)
router_topk_kernel(const double *__restrict__ logits, int E, int k, const uint16_t *__restrict__ pes,
                   int32_t *__restrict__ idx, float *__restrict__ wts) {
    __shared__ double v[kMaxE];
    __shared__ unsigned char taken[kMaxE];
    __shared__ double selv[kMaxK];
    __shared__ int sel[kMaxK];
    const int t = blockIdx.x, lane = threadIdx.x;
    for (int e = lane; e < E; e += kWarp) {
        v[e] = logits[(size_t)t * E + e];
        taken[e] = 0;
    }
    __syncwarp();
    for (int s = 0; s < k; ++s) {
        double bv = 0.0;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += kWarp) {
            if (taken[e]) continue;
            const double x = v[e];
            if (be == 0x7fffffff || x > bv || (x == bv && e < be)) {
                bv = x;
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if (lane == 0) {
            taken[be] = 1;
            sel[s] = be;
            selv[s] = bv;
        }
        __syncwarp();
    }
    // softmax over the selected logits; selv[0] is their maximum
    const double p = lane < k ? exp(selv[lane] - selv[0]) : 0.0;
    const double z = warp_sum(p);
    if (lane < k) {
        idx[(size_t)t * k + lane] = sel[lane];
        wts[(size_t)t * k + lane] = (float)(p / z * (double)bf16_bits_to_float(pes[sel[lane]]));
    }
}

size_t router_logits_smem(int H) {
    const size_t nchunk = (size_t)H / 16;
    return sizeof(double) * (16 * (nchunk | 1) + nchunk + kRouterRows);
}

cudaError_t launch_router_logits(const moe_layer_w *w, const uint16_t *h, int T, float eps, double *logits,
                                 uint16_t *xe, cudaStream_t st) {
    const size_t smem = router_logits_smem(w->H);
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(router_logits_kernel), smem);
    if (e != cudaSuccess) return e;
    // many tokens: one CTA covers 32 experts (the token's norm is computed
    // once for them); few tokens: 8, so that more CTAs share the work
    const int epw = T >= 16 ? 4 : 1;
    dim3 grid((w->E + kRouterRows * epw - 1) / (kRouterRows * epw), T);
    router_logits_kernel<<<grid, kRouterThreads, smem, st>>>(w->router_q, w->router_s, w->router_b,
                                                             w->router_scale, h, w->H, w->E, epw, eps, logits, xe);
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const double *logits, int T, int E, int k, const uint16_t *pes, int32_t *idx,
                               float *wts, cudaStream_t st) {
    router_topk_kernel<<<T, kWarp, 0, st>>>(logits, E, k, pes, idx, wts);
    return cudaGetLastError();
}

}  // namespace moe
