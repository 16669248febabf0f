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

// The same logits for many tokens: a CTA takes kRtTok tokens and 32 experts,
// each warp 4 experts for all kRtTok tokens, so a code is read and turned
// into a double once for kRtTok products and a staged input once for 4
// experts.  The norm, the staging and the per-chunk order of the sums are the
// one-token kernel's.
constexpr int kRtTok = 4;  // tokens per CTA
constexpr int kRtEpw = 4;  // experts per warp

__global__ void __launch_bounds__(kRouterThreads)
router_logits_tiled_kernel(const uint32_t *__restrict__ rq, const uint16_t *__restrict__ rs,
                           const uint16_t *__restrict__ rb, const uint16_t *__restrict__ router_scale,
                           const uint16_t *__restrict__ h, int H, int E, int T, float eps,
                           double *__restrict__ logits, uint16_t *__restrict__ xe) {
    extern __shared__ double smem_d[];
    const int nchunk = H / 16;
    const int ld = nchunk | 1;
    double *xsT = smem_d;                                    // [kRtTok][16][ld]
    double *csum = xsT + (size_t)kRtTok * 16 * ld;           // [kRtTok][nchunk]
    double *red = csum + (size_t)kRtTok * nchunk;            // [kRouterRows]
    const int t0 = blockIdx.y * kRtTok, nt = min(kRtTok, T - t0);
    const double inv_sqrt_h = 1.0 / sqrt((double)H);
    const bool write_xe = (xe != nullptr) && blockIdx.x == 0;
    const int lane = threadIdx.x & 31;
    const int G = H / kGroup;
    const int e0 = (blockIdx.x * kRouterRows + (threadIdx.x >> 5)) * kRtEpw;
    // a chunk's codes and its group's (scale, bias) for the warp's experts, one chunk ahead; the
    // first chunk's are asked for before the norm
    uint4 qc[kRtEpw], qn[kRtEpw];
    uint32_t sbc[kRtEpw], sbn[kRtEpw];
    auto load = [&](int c, uint4 (&q)[kRtEpw], uint32_t (&sb)[kRtEpw]) {
#pragma unroll
        for (int x = 0; x < kRtEpw; ++x) {
            const int e = min(e0 + x, E - 1);
            q[x] = ldg_nc_v4(rq + (size_t)e * (H / 4) + 4 * c);
            sb[x] = (uint32_t)__ldg(rs + (size_t)e * G + (c >> 2)) | ((uint32_t)__ldg(rb + (size_t)e * G + (c >> 2)) << 16);
        }
    };
    if (e0 < E && lane < nchunk) load(lane, qc, sbc);
    // the tokens' sums of squares over 8-element packs, every token's loads in flight together
    const int npk = H / 8;
    double ss[kRtTok];
#pragma unroll
    for (int j = 0; j < kRtTok; ++j) ss[j] = 0.0;
    for (int p = threadIdx.x; p < npk; p += blockDim.x) {
        uint4 v[kRtTok];
#pragma unroll
        for (int j = 0; j < kRtTok; ++j)
            v[j] = j < nt ? __ldg(reinterpret_cast<const uint4 *>(h + (size_t)(t0 + j) * H) + p) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < kRtTok; ++j) {
            const uint32_t wv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const double d = (double)bf16_bits_to_float((wv[q >> 1] >> (16 * (q & 1))) & 0xffffu);
                ss[j] += d * d;
            }
        }
    }
    double rinv[kRtTok];
#pragma unroll
    for (int j = 0; j < kRtTok; ++j) {
        rinv[j] = 0.0;
        if (j < nt) rinv[j] = 1.0 / sqrt(block_sum(ss[j], red) / (double)H + (double)eps);
    }
    for (int p = threadIdx.x; p < npk; p += blockDim.x) {
        const uint4 rv = __ldg(reinterpret_cast<const uint4 *>(router_scale) + p);
        const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
        uint4 v[kRtTok];
#pragma unroll
        for (int j = 0; j < kRtTok; ++j)
            v[j] = j < nt ? __ldg(reinterpret_cast<const uint4 *>(h + (size_t)(t0 + j) * H) + p) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < kRtTok; ++j) {
            if (j >= nt) break;
            const uint32_t wv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t ob[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = 8 * p + q;
                const double xn = (double)bf16_bits_to_float((wv[q >> 1] >> (16 * (q & 1))) & 0xffffu) * rinv[j];
                const double xs = xn * (double)bf16_bits_to_float((rw[q >> 1] >> (16 * (q & 1))) & 0xffffu) * inv_sqrt_h;
                xsT[((size_t)j * 16 + (i & 15)) * ld + (i >> 4)] = xs;
                ob[q] = f64_to_bf16_bits(xn);
            }
            if (write_xe)
                reinterpret_cast<uint4 *>(xe + (size_t)(t0 + j) * H)[p] =
                    make_uint4(ob[0] | (ob[1] << 16), ob[2] | (ob[3] << 16), ob[4] | (ob[5] << 16), ob[6] | (ob[7] << 16));
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nt * nchunk; i += blockDim.x) {
        const int j = i / nchunk, c = i - j * nchunk;
        double s = 0.0;
#pragma unroll
        for (int m = 0; m < 16; ++m) s += xsT[((size_t)j * 16 + m) * ld + c];
        csum[(size_t)j * nchunk + c] = s;
    }
    __syncthreads();

    double acc[kRtTok][kRtEpw];
#pragma unroll
    for (int j = 0; j < kRtTok; ++j)
#pragma unroll
        for (int x = 0; x < kRtEpw; ++x) acc[j][x] = 0.0;
    if (e0 < E) {
        for (int c = lane; c < nchunk; c += kWarp) {
            if (c + kWarp < nchunk) load(c + kWarp, qn, sbn);
            double dot[kRtTok][kRtEpw];
#pragma unroll
            for (int j = 0; j < kRtTok; ++j)
#pragma unroll
                for (int x = 0; x < kRtEpw; ++x) dot[j][x] = 0.0;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                double xv[kRtTok];
#pragma unroll
                for (int j = 0; j < kRtTok; ++j) xv[j] = j < nt ? xsT[((size_t)j * 16 + m) * ld + c] : 0.0;
#pragma unroll
                for (int x = 0; x < kRtEpw; ++x) {
                    const uint32_t wd = m < 4 ? qc[x].x : m < 8 ? qc[x].y : m < 12 ? qc[x].z : qc[x].w;
                    // the 8-bit code as a double: 2^52 + q read as fp64, minus 2^52
                    const double qd =
                        __hiloint2double(0x43300000, (int)((wd >> (8 * (m & 3))) & 0xffu)) - 4503599627370496.0;
#pragma unroll
                    for (int j = 0; j < kRtTok; ++j) dot[j][x] += qd * xv[j];
                }
            }
#pragma unroll
            for (int x = 0; x < kRtEpw; ++x) {
                const double sc = (double)bf16_bits_to_float(sbc[x] & 0xffffu);
                const double bi = (double)bf16_bits_to_float(sbc[x] >> 16);
#pragma unroll
                for (int j = 0; j < kRtTok; ++j)
                    acc[j][x] += sc * dot[j][x] + bi * (j < nt ? csum[(size_t)j * nchunk + c] : 0.0);
            }
#pragma unroll
            for (int x = 0; x < kRtEpw; ++x) {
                qc[x] = qn[x];
                sbc[x] = sbn[x];
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kRtTok; ++j)
#pragma unroll
        for (int x = 0; x < kRtEpw; ++x) {
            const double v = warp_sum(acc[j][x]);
            if (lane == 0 && j < nt && e0 + x < E) logits[(size_t)(t0 + j) * E + e0 + x] = v;
        }
}

// The logit as an order-preserving 64-bit key (larger logit <=> larger key;
// -0 and +0 are the same logit).
__device__ __forceinline__ unsigned long long topk_key(double v) {
    unsigned long long b = (unsigned long long)__double_as_longlong(v);
    if (b == 0x8000000000000000ull) b = 0ull;
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double topk_logit(unsigned long long k) {
    const unsigned long long b = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double((long long)b);
}

// One warp per token, lane j holding the keys of experts j, 32 + j, ... in
// registers.  k rounds: every lane offers its largest key not yet taken (the
// lower expert on equal keys), two 32-bit max-reductions (high word, then low
// word among the lanes holding the high word) give the largest key and a
// min-reduction the lowest expert holding it; ordered by (logit desc, index
// asc).  Then the softmax over the k selected logits in fp64, times
// per_expert_scale.
template <int NSL>
__global__ void __launch_bounds__(kWarp)
router_topk_kernel(const double *__restrict__ logits, int E, int k, const uint16_t *__restrict__ pes,
                   int32_t *__restrict__ idx, float *__restrict__ wts) {
    __shared__ double selv[kMaxK];
    __shared__ int sel[kMaxK];
    const int t = blockIdx.x, lane = threadIdx.x;
    unsigned long long key[NSL];
#pragma unroll
    for (int sl = 0; sl < NSL; ++sl) {
        const int e = sl * kWarp + lane;
        key[sl] = e < E ? topk_key(logits[(size_t)t * E + e]) : 0ull;  // 0: below every logit's key
    }
    for (int s = 0; s < k; ++s) {
        unsigned long long best = 0ull;
        int bsl = 0;
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl)
            if (key[sl] > best) {  // strict: the lower expert on equal keys
                best = key[sl];
                bsl = sl;
            }
        const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(best >> 32));
        const unsigned lo = __reduce_max_sync(0xffffffffu, (unsigned)(best >> 32) == hi ? (unsigned)best : 0u);
        const unsigned long long top = ((unsigned long long)hi << 32) | lo;
        const unsigned e = __reduce_min_sync(0xffffffffu, best == top ? (unsigned)(bsl * kWarp + lane) : 0xffffffffu);
        if (lane == (int)(e & 31u)) {
#pragma unroll
            for (int sl = 0; sl < NSL; ++sl)
                if (sl == bsl) key[sl] = 0ull;
        }
        if (lane == 0) {
            sel[s] = (int)e;
            selv[s] = topk_logit(top);
        }
    }
    __syncwarp();
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

size_t router_logits_tiled_smem(int H) {
    const size_t nchunk = (size_t)H / 16;
    return sizeof(double) * (kRtTok * 16 * (nchunk | 1) + kRtTok * nchunk + kRouterRows);
}

cudaError_t launch_router_logits(const moe_layer_w *w, const uint16_t *h, int T, float eps, double *logits,
                                 uint16_t *xe, cudaStream_t st) {
    if (T >= 16) {  // many tokens: tiles of kRtTok tokens x 32 experts
        const size_t smem = router_logits_tiled_smem(w->H);
        cudaError_t e = ensure_smem(reinterpret_cast<const void *>(router_logits_tiled_kernel), smem);
        if (e != cudaSuccess) return e;
        dim3 grid((w->E + kRouterRows * kRtEpw - 1) / (kRouterRows * kRtEpw), (T + kRtTok - 1) / kRtTok);
        router_logits_tiled_kernel<<<grid, kRouterThreads, smem, st>>>(
            w->router_q, w->router_s, w->router_b, w->router_scale, h, w->H, w->E, T, eps, logits, xe);
        return cudaGetLastError();
    }
    const size_t smem = router_logits_smem(w->H);
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(router_logits_kernel), smem);
    if (e != cudaSuccess) return e;
    // few tokens: one CTA per token and 8 experts, so that more CTAs share the work
    const int epw = 1;
    dim3 grid((w->E + kRouterRows * epw - 1) / (kRouterRows * epw), T);
    router_logits_kernel<<<grid, kRouterThreads, smem, st>>>(w->router_q, w->router_s, w->router_b,
                                                             w->router_scale, h, w->H, w->E, epw, eps, logits, xe);
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const double *logits, int T, int E, int k, const uint16_t *pes, int32_t *idx,
                               float *wts, cudaStream_t st) {
    if (E <= 4 * kWarp) router_topk_kernel<4><<<T, kWarp, 0, st>>>(logits, E, k, pes, idx, wts);
    else if (E <= 8 * kWarp) router_topk_kernel<8><<<T, kWarp, 0, st>>>(logits, E, k, pes, idx, wts);
    else if (E <= 16 * kWarp) router_topk_kernel<16><<<T, kWarp, 0, st>>>(logits, E, k, pes, idx, wts);
    else router_topk_kernel<32><<<T, kWarp, 0, st>>>(logits, E, k, pes, idx, wts);
    return cudaGetLastError();
}

}  // namespace moe
