// moe_cache.cu -- tiered expert residency: the routed experts of a layer live
// in a pool in host memory, and a cache of C experts per layer in device
// memory holds the ones in use.
//
// TurboFieldfare introduction page (discuss.pytorch.kr), section
// "TurboFieldfare's expert streaming structure": per layer, a 16-slot LFU
// cache of experts; after the router, hits are served from it and only the
// misses are read (there from SSD with parallel reads, overlapped with the
// shared expert).  Swiftlet article (tech.utomolab.com), section "why the
// same model runs in so little memory": an LFU + recency cache pool.  Here
// the pool is host memory that the GPU reads over the bus, the cache is HBM,
// and every decision stays on the GPU: no routing result goes back to the
// host.
//
//   residency_kernel  one CTA: for the distinct experts the call selected, in
//                     ascending expert order: a hit counts a use; a miss takes
//                     the slot with the fewest uses among those the call does
//                     not need (ties: least recently used, then the lowest
//                     slot; empty slots first), and is listed for the copy.
//                     Then every pair's expert id becomes its slot id.
//   fill_kernel       copies the listed experts' gate, up and down matrices
//                     (codes and scale/bias words) from the pool into their
//                     slots, 16 bytes per thread and step, all CTAs over the
//                     concatenated bytes of every miss.
// The layer then runs bucketing and the expert FFN on the cache as if it
// had C experts; the router and gate weights use the real expert ids.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kResThreads = 256;

__global__ void __launch_bounds__(kResThreads)
residency_kernel(const int32_t *__restrict__ idx, int n, int E, int C, int32_t *__restrict__ slot_of,
                 int32_t *__restrict__ expert_of, uint32_t *__restrict__ uses, uint32_t *__restrict__ last,
                 uint32_t *__restrict__ ctl, int32_t *__restrict__ miss, int32_t *__restrict__ idx_c) {
    extern __shared__ unsigned char res_smem[];
    unsigned char *needed = res_smem;              // [E]
    unsigned char *pinned = res_smem + E;          // [C]
    for (int e = threadIdx.x; e < E; e += blockDim.x) needed[e] = 0;
    for (int s = threadIdx.x; s < C; s += blockDim.x) pinned[s] = 0;
    __syncthreads();
    for (int p = threadIdx.x; p < n; p += blockDim.x) needed[idx[p]] = 1;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (needed[e] && slot_of[e] >= 0) pinned[slot_of[e]] = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t tick = ctl[0] + 1u;
        uint32_t hits = 0, misses = 0;
        int nm = 0;
        for (int e = 0; e < E; ++e) {
            if (!needed[e]) continue;
            int s = slot_of[e];
            if (s >= 0) {
                ++hits;
                uses[s] += 1u;
                last[s] = tick;
                continue;
            }
            // victim: an empty slot first, else the fewest uses, then the oldest use, then the lowest slot
            int v = -1;
            for (int c = 0; c < C; ++c) {
                if (pinned[c]) continue;
                if (v < 0) {
                    v = c;
                    continue;
                }
                const bool ce = expert_of[c] < 0, ve = expert_of[v] < 0;
                if (ce != ve) {
                    if (ce) v = c;
                    continue;
                }
                if (ce) continue;  // both empty: keep the lower slot
                if (uses[c] < uses[v] || (uses[c] == uses[v] && last[c] < last[v])) v = c;
            }
            // v >= 0: the host checked C >= the distinct experts one call can select
            if (expert_of[v] >= 0) slot_of[expert_of[v]] = -1;
            expert_of[v] = e;
            slot_of[e] = v;
            uses[v] = 1u;
            last[v] = tick;
            pinned[v] = 1;
            miss[1 + 2 * nm] = e;
            miss[2 + 2 * nm] = v;
            ++nm;
            ++misses;
        }
        miss[0] = nm;
        ctl[0] = tick;
        ctl[1] += hits;
        ctl[2] += misses;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < n; p += blockDim.x) idx_c[p] = slot_of[idx[p]];
}

struct FillArgs {
    const uint4 *src[6];  // pool: gate q, gate sb, up q, up sb, down q, down sb (expert 0)
    uint4 *dst[6];        // cache (slot 0)
    long long per[6];     // 16-byte units per expert of each array
    long long total;      // units per expert over the six arrays
};

// Copies every listed miss (expert e -> slot v) from the pool to the cache.
__global__ void __launch_bounds__(256) fill_kernel(FillArgs a, const int32_t *__restrict__ miss) {
    const int nm = miss[0];
    const long long all = (long long)nm * a.total;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < all;
         i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / a.total);
        long long r = i - (long long)m * a.total;
        int k = 0;
        while (r >= a.per[k]) {
            r -= a.per[k];
            ++k;
        }
        const int e = miss[1 + 2 * m], v = miss[2 + 2 * m];
        a.dst[k][(long long)v * a.per[k] + r] = a.src[k][(long long)e * a.per[k] + r];
    }
}

cudaError_t launch_residency(const int32_t *idx, int n, int E, int C, int32_t *slot_of, int32_t *expert_of,
                             uint32_t *uses, uint32_t *last, uint32_t *ctl, int32_t *miss, int32_t *idx_c,
                             cudaStream_t st) {
    residency_kernel<<<1, kResThreads, (size_t)E + (size_t)C, st>>>(idx, n, E, C, slot_of, expert_of, uses, last, ctl,
                                                                      miss, idx_c);
    return cudaGetLastError();
}

cudaError_t launch_fill(const moe_layer_w *w, const moe_qmat pool[3], const moe_qmat cache[3], const int32_t *miss,
                        cudaStream_t st) {
    const long long H = w->H, I = w->I;
    FillArgs a;
    const long long q_gu = I * H / 2 / 16, sb_gu = I * (H / 64) * 4 / 16;  // per expert, 16-byte units
    const long long q_d = H * I / 2 / 16, sb_d = H * (I / 64) * 4 / 16;
    const long long per[6] = {q_gu, sb_gu, q_gu, sb_gu, q_d, sb_d};
    for (int m = 0; m < 3; ++m) {
        a.src[2 * m] = reinterpret_cast<const uint4 *>(pool[m].q);
        a.src[2 * m + 1] = reinterpret_cast<const uint4 *>(pool[m].sb);
        a.dst[2 * m] = reinterpret_cast<uint4 *>(const_cast<uint32_t *>(cache[m].q));
        a.dst[2 * m + 1] = reinterpret_cast<uint4 *>(const_cast<uint32_t *>(cache[m].sb));
    }
    a.total = 0;
    for (int k = 0; k < 6; ++k) {
        a.per[k] = per[k];
        a.total += per[k];
    }
    int dev = 0, sms = 0;
    cudaError_t e = stream_device(st, &dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    fill_kernel<<<2 * sms, 256, 0, st>>>(a, miss);
    return cudaGetLastError();
}

__global__ void cache_reset_kernel(int E, int C, int32_t *slot_of, int32_t *expert_of, uint32_t *uses, uint32_t *last,
                                   uint32_t *ctl) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < E || i < C || i < 4; i += gridDim.x * blockDim.x) {
        if (i < E) slot_of[i] = -1;
        if (i < C) {
            expert_of[i] = -1;
            uses[i] = 0u;
            last[i] = 0u;
        }
        if (i < 4) ctl[i] = 0u;
    }
}

cudaError_t launch_cache_reset(int E, int C, int32_t *slot_of, int32_t *expert_of, uint32_t *uses, uint32_t *last,
                               uint32_t *ctl, cudaStream_t st) {
    cache_reset_kernel<<<4, 256, 0, st>>>(E, C, slot_of, expert_of, uses, last, ctl);
    return cudaGetLastError();
}

}  // namespace moe
