// moe_bucket.cu -- token -> expert bucketing.
//
// The (token, slot) pairs of a call are grouped by expert so that one read of
// an expert's weights serves every row routed to it (the reason the
// TurboFieldfare page gives for chunked prefill, section "TurboFieldfare's
// expert streaming structure", last paragraph).  Output: offsets[E+1]
// (exclusive prefix sum of pairs per expert), perm (pair ids t*k+s grouped by
// expert, ascending inside an expert), inv (inv[perm[j]] = j) and the list of
// experts that received at least one pair.  Integer-only and deterministic.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kBucketThreads = 256;
constexpr int kBucketWarps = kBucketThreads / kWarp;

// Warp w owns a contiguous block of the pairs.  Counting per (warp, expert)
// and an exclusive sum over the warps give each warp the first position of
// its block's pairs inside every expert's segment, so the 8 warps scatter at
// once and the result is the same stable order (by expert, then pair id) as
// one pass over all pairs.
__global__ void __launch_bounds__(kBucketThreads)
bucket_kernel(const int32_t *__restrict__ idx, int n, int E, int32_t *__restrict__ offsets,
              int32_t *__restrict__ perm, int32_t *__restrict__ inv, int32_t *__restrict__ active) {
    __shared__ int cnt[kMaxE];
    __shared__ int cursor[kMaxE];
    __shared__ int wpos[kBucketWarps][kMaxE];  // per warp and expert: its count, then its first position
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int e = tid; e < E; e += blockDim.x)
        for (int w = 0; w < kBucketWarps; ++w) wpos[w][e] = 0;
    __syncthreads();
    const int B = ((n + kBucketWarps - 1) / kBucketWarps + kWarp - 1) & ~(kWarp - 1);
    const int p0 = min(n, wid * B), p1 = min(n, p0 + B);
    for (int p = p0 + lane; p < p1; p += kWarp) {
        const int e = idx[p];
        if (e >= 0 && e < E) atomicAdd(&wpos[wid][e], 1);  // integer counts: order does not matter
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kBucketWarps; ++w) {
            const int c = wpos[w][e];
            wpos[w][e] = run;
            run += c;
        }
        cnt[e] = run;
    }
    __syncthreads();
    if (wid == 0) {
        // exclusive scan of the counts and the compacted list of used experts
        int run = 0, nact = 0;
        for (int base = 0; base < E; base += kWarp) {
            const int e = base + lane;
            const int c = e < E ? cnt[e] : 0;
            int inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            const unsigned used = __ballot_sync(0xffffffffu, c > 0);
            if (e < E) {
                offsets[e] = run + inc - c;
                cursor[e] = run + inc - c;
                if (active && c > 0) active[1 + nact + __popc(used & ((1u << lane) - 1u))] = e;
            }
            run += __shfl_sync(0xffffffffu, inc, 31);
            nact += __popc(used);
        }
        if (lane == 0) {
            offsets[E] = run;
            if (active) active[0] = nact;
        }
    }
    __syncthreads();
    // stable scatter of this warp's block, 32 pairs at a time in ascending pair order
    for (int base = p0; base < p1; base += kWarp) {
        const int p = base + lane;
        int e = p < p1 ? idx[p] : -1;
        const bool ok = e >= 0 && e < E;
        if (!ok) e = -2 - lane;  // unique key: never matches a real expert
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (ok) {
            const int pos = cursor[e] + wpos[wid][e] + rank;
            perm[pos] = p;
            if (inv) inv[p] = pos;
        }
        __syncwarp();
        if (ok && rank == 0) wpos[wid][e] += __popc(peers);
        __syncwarp();
    }
}

cudaError_t launch_bucket(const int32_t *idx, int n_pairs, int E, int32_t *offsets, int32_t *perm, int32_t *inv,
                          int32_t *active, cudaStream_t st) {
    bucket_kernel<<<1, kBucketThreads, 0, st>>>(idx, n_pairs, E, offsets, perm, inv, active);
    return cudaGetLastError();
}

}  // namespace moe
