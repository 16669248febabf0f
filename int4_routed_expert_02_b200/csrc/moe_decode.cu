// moe_decode.cu -- persistent decode kernel: a stack of MoE layers for a small
// token batch (T <= 8) in ONE cooperative launch, one CTA per SM.
//
// Per layer (TurboFieldfare introduction page, discuss.pytorch.kr, section
// "TurboFieldfare's expert streaming structure": router -> routed experts +
// shared expert -> weighted combine -> normalisation, residual, layer scalar;
// weights MLX affine, section "How TurboFieldfare saves memory"), one layer is
// a chain of three grid-wide exchanges and the weight streams between them:
//
//   F  every CTA reads the previous layer's combine m (all rows), finishes that
//      layer (post-norm, residual, layer scalar; CTA c writes its slice of the
//      bf16 output) and forms this layer's expert input xe = bf16(rmsnorm(h)),
//      pre-scaled for the code decode
//   R  router logits in fp64 for this CTA's share of the experts, into global
//      memory as flag-in-data words (each carries the layer's tag)
//   S  the shared expert's gate/up rows of this CTA (they need only xe): each
//      8-row unit is 8 one-row pieces, one warp each; a piece forms the row's
//      g and u over the whole input and a = silu(g) * u, stored in global
//      memory; the last piece of a unit counts the unit done (release)
//   K  read every logit, polling each until it carries this layer's tag (no
//      barrier); top-k (ties to the lower index) and
//      softmax * per_expert_scale, redundantly on every CTA, and the
//      bucketing of the T*k pairs into distinct experts ("slots")
//   G  routed gate/up units (slot, 8 rows), dealt round-robin over the grid
//      in slot order, so that early slots complete early; pieces as in S
//   D  down projection of this CTA's output rows (8-row blocks): per slot, as
//      soon as that slot's a is complete everywhere (its unit count), the
//      first warp stages a into the slot's ring slot and the block tasks run
//      -- so the down of early slots overlaps the gate/up of later ones
//   then the CTA sums its rows' routed outputs with the gate weights and the
//      shared output in a fixed order (deterministic), writes m, and arrives
//      at the next layer's barrier.
//
// Weights move HBM -> shared memory by TMA tensor copies (no multicast) into a
// ring of fixed-size slots, issued by one producer thread ahead of 15
// consumer warps.  Once the top-k is known the producer asks L2 to prefetch
// every routed byte this CTA will need (and, after the routed units, the next
// layer's router and shared-expert units), so HBM streams across the
// exchanges while the ring fills in order.  The 4-bit codes are decoded with
// the subnormal trick of moe_common.cuh (one AND and half a packed FMA per
// code against inputs pre-scaled per nibble position); products are exact and
// sums fp32.  The router accumulates in fp64 so that the top-k does not depend
// on the summation order.
//
// Every wait (grid barriers, readiness counts, mbarriers, slot ownership) is
// bounded by ~1 s of globaltimer; on a timeout the kernel records an error
// code in the workspace, every CTA stops taking work, the producer lets its
// own copies land, and the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace dec {

constexpr int kCW = 15;                       // consumer warps
constexpr int kProdWarp = kCW;                // the producer warp (its lane 0 issues every copy)
constexpr int kThreads = (kCW + 1) * 32;      // 512: 4 warps per SM sub-partition, 128 registers a thread
constexpr int kCThreads = kCW * 32;
constexpr int kMaxT = 8;
constexpr int kMaxLayers = 64;
constexpr int kMaxPairs = kMaxT * kMaxK;      // 256
constexpr int kMaxSlots = 16;                 // ring slots
constexpr int kMaxA = 9;                      // the static region's tasks: router rows + up to 8 shared units
constexpr int kXmBlk = 8;                     // expert-major down items: 8-row blocks per item (a multiple of 4)
constexpr int kMaxStage = 3;                  // expert-major down: experts whose SwiGLU input a CTA stages per layer
constexpr int kMaps = 12;                     // TMA tensor maps per layer
constexpr int kMaxBlk = 4;                    // 8-row output blocks per CTA (H <= 4096 on >= 128 SMs)
constexpr int kMaxParts = 8;                  // K-parts of a down matrix
constexpr int kPartChunks = 32;               // at most 32 chunks (1024 columns) per K-part
constexpr int kBarCtrs = 1;                   // grid-barrier counters, 128 bytes apart (one polls fastest)
constexpr int kMaxStageTH = 24576;            // largest T * H
constexpr int kMaxSl = 16;                    // groups of 32 experts (E <= 512)
constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s

enum { kErrBarrier = 1, kErrFull, kErrEmpty, kErrReady, kErrOwner, kErrTables, kErrStage, kErrLogits };
enum {
    kMapGateQ = 0, kMapUpQ, kMapGateSb, kMapUpSb,        // routed gate/up: codes, (scale, bias) words
    kMapShGateQ, kMapShUpQ, kMapShGateSb, kMapShUpSb,    // shared gate/up
    kMapDownQ, kMapDownSb, kMapShDownQ, kMapShDownSb     // routed and shared down
};

// Sizes, options, shared-memory plan and workspace pointers of a launch.
// Copied into shared memory at the start, so phases read them at shared
// latency instead of through the parameter space.
struct Cfg {
    const uint16_t *h_in;  // chained: [T,H]; else [L,T,H]
    uint16_t *h_out;       // [L,T,H]: every layer's output
    int L, T, chained, post_norm;
    float layer_scalar, eps;
    int H, E, k, I, Is;
    int CH, GH;                  // 32-column chunks and 64-column groups of H
    int units_s, units_r;        // 8-row units of the shared / one routed gate (or up) matrix
    int nrb8;                    // 8-row blocks of the output rows (H / 8)
    int parts_s, pc_s;           // shared down: K-parts, chunks per part
    int parts_r, pc_r;           // routed down
    int ns, slot_bytes;          // ring slots and their size (routed gate/up units and down groups)
    int a_rbytes, a_ubytes;      // static region: router part, one shared gate/up unit (1024-aligned)
    int ua;                      // shared units a CTA keeps in the static region (the rest go through the ring)
    int gcb;                     // bytes of one matrix's codes in a gate/up slot (1024-aligned)
    int sbs;                     // bytes of one matrix's (scale, bias) words in a gate/up slot (128-aligned)
    int dcb_s, dcb_r;            // bytes of one 8-row block's codes in a down slot (1024-aligned)
    int sbd_s, sbd_r;            // bytes of one 8-row block's words in a down slot (128-aligned)
    int off_a, off_ring, off_x, off_xs, off_h, off_y, off_part;  // dynamic shared memory offsets
    int yrows;                   // rows per ybuf entry (8 * kMaxBlk)
    unsigned *bar;               // [kBarCtrs * 32] monotonic arrival counters
    unsigned bar_extra;          // arrivals beyond the grid the barriers wait for (tests of the timeout path)
    int *err;                    // device status word
    unsigned *ready;             // [1 + kMaxPairs]: gate/up units done, shared then per routed slot
    unsigned long long *logit_ll;  // [T,E][2]: each logit as two words (32 bits of it | layer tag << 32)
    float *a_sh;                 // [T,Is]   SwiGLU output of the shared expert
    float *a_r;                  // [T*k,I]  of the routed experts, by bucketed position
    float *m;                    // [T,H]    combine of the current layer
    const CUtensorMap *maps;     // [L][kMaps]
    int xm;                      // tensor-core variant: routed down work by expert (see consumer_main)
    int ipe;                     // expert-major down items per expert (H / (8 kXmBlk))
    int stage_bytes, off_stage;  // expert-major down: one expert's staged input, and where they sit
    int nstage;                  // expert-major down: staged experts a CTA has room for (<= kMaxStage)
    float *y_r;                  // [T*k,H]  expert-major down: routed outputs by pair id
};

struct Params {
    Cfg c;
    moe_layer_w layers[kMaxLayers];
};

// Fixed part of the shared memory (at its 1024-aligned base).
struct Shared {
    unsigned long long full[kMaxSlots];    // ring slot filled (TMA completion)
    unsigned long long empty[kMaxSlots];   // ring slot consumed
    volatile unsigned owner[kMaxSlots];    // sequence number of the task a slot holds
    int cnt[kMaxSlots];                    // pieces / block tasks of the slot's task that are done
    volatile int astate[kMaxSlots];        // down slot: 0 a not staged, 1 staging, 2 staged
    unsigned long long afull[kMaxA];       // static region task filled (phase = layer parity)
    unsigned long long aempty;             // static region consumed (1 + shared units arrivals per layer)
    int acnt[kMaxA];                       // pieces of a shared unit that are done
    volatile int tables_layer;             // 1 + the layer whose routing tables are ready
    volatile int verdict;                  // consumers: 1 while no error is recorded
    volatile int kverdict;                 // the token warps' verdict on this layer's routing
    int D;                                 // distinct experts of the current layer
    int slot_e[kMaxPairs], slot_off[kMaxPairs], slot_n[kMaxPairs];
    int pos_tok[kMaxPairs];                // bucketed position -> token
    int pos_pair[kMaxPairs];               // bucketed position -> pair id t*k + s
    int pos_idx[kMaxPairs];                // 0, 1, 2, ...: bucketed positions (rows of the routed SwiGLU buffer)
    int first[kMaxPairs];                  // pair is the first of its expert
    int idx[kMaxPairs];                    // [t][s] selected expert
    double selv[kMaxPairs];                // [t][s] its logit
    float wts[kMaxPairs];                  // [t][s] gate weight
    unsigned exp_ready[1 + kMaxPairs];     // readiness counts expected once this layer's units are done
    float rms[kMaxT], rinv[kMaxT];
    float red[32];
    double rpart[kCW];                     // router partial sums (fewer items than warps)
    int toks_sh[kMaxT];                    // 0, 1, ..., T-1
    Cfg c;
    volatile int xstate[kMaxStage];        // expert-major down: as astate, for each staged expert
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(unsigned long long *b, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long *b, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_test(unsigned long long *b, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ int ldcg_int(const int *p) { return __ldcg(p); }

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for the phase with `parity` of mbarrier `b`; false on a timeout
// (recorded with `code`) or when an error is already recorded.
__device__ __noinline__ bool mbar_wait(unsigned long long *b, unsigned parity, int *err, int code) {
    if (mbar_test(b, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 1;; ++it) {
        if (mbar_test(b, parity)) return true;
        if ((it & 63u) == 0) {
            if (ldcg_int(err) != 0) return false;
            if (globaltimer() - t0 > kWaitNs) {
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// Bounded wait used when stopping: ignores the error word.
__device__ __noinline__ void mbar_drain(unsigned long long *b, unsigned parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_test(b, parity)) {
        if (globaltimer() - t0 > kWaitNs) return;
    }
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, unsigned bytes, unsigned long long *b) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(b))
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *src, unsigned bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 3-D tiled TMA load (no multicast) of the box at (x, y, z) of `map`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            unsigned long long *b) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(b))
        : "memory");
}

// The descriptor of a tensor map into the TMA unit's cache ahead of its first use.
__device__ __forceinline__ void prefetch_map(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// The same box into L2 only.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(x), "r"(y),
                 "r"(z)
                 : "memory");
}

// Named barrier of the 15 consumer warps.
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCThreads) : "memory"); }

// Named barrier of the T token warps (the top-k and the buckets).
__device__ __forceinline__ void token_warps_sync(int T) { asm volatile("bar.sync 2, %0;" ::"r"(T * 32) : "memory"); }

// ------------------------------------------------------------------ grid barrier (split phase)

// Arrival of this CTA (thread 0 of the consumers, after a consumer barrier):
// its global writes become visible before the count.
__device__ __forceinline__ void grid_arrive(const Cfg &P) {
    __threadfence();
    red_release_add(P.bar + 32 * (blockIdx.x % kBarCtrs), 1u);
}

// Wait until every CTA has arrived `nth` times (sum of the counters); called
// by all consumer threads.  False (uniformly) if an error is recorded.
__device__ __noinline__ bool grid_wait(const Cfg &P, Shared &S, unsigned nth) {
    consumer_sync();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const unsigned target = nth * gridDim.x + P.bar_extra;
        const unsigned long long t0 = globaltimer();
        bool ok = true;
        for (unsigned it = 0;; ++it) {
            unsigned v = lane < kBarCtrs ? ld_acquire(P.bar + 32 * lane) : 0u;
            // the full butterfly: every lane holds the same sum, so all lanes leave the loop together
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (v >= target) break;
            if ((it & 63u) == 63u) {
                int bad = 0;
                if (lane == 0) {
                    bad = ldcg_int(P.err) != 0;
                    if (!bad && globaltimer() - t0 > kWaitNs) {
                        atomicCAS(P.err, 0, kErrBarrier);
                        bad = 1;
                    }
                }
                if (__shfl_sync(0xffffffffu, bad, 0)) {
                    ok = false;
                    break;
                }
            }
        }
        __threadfence();
        if (lane == 0) S.verdict = ok && ldcg_int(P.err) == 0;
    }
    consumer_sync();
    return S.verdict != 0;
}

// Bounded wait of lane 0 until a global count reaches `target` (acquire).
__device__ __noinline__ bool wait_count(const Cfg &P, const unsigned *ctr, unsigned target) {
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 0;; ++it) {
        if (ld_acquire(ctr) >= target) return true;
        if ((it & 63u) == 63u) {
            if (ldcg_int(P.err) != 0) return false;
            if (globaltimer() - t0 > kWaitNs) {
                atomicCAS(P.err, 0, kErrReady);
                return false;
            }
        }
        __nanosleep(32);
    }
}

// The logits exchange carries its own validity: a logit is written as two
// 8-byte words, each holding 32 bits of it and the layer's tag (1 + layer)
// above them.  An aligned 8-byte store is seen whole or not at all, so a
// reader that finds the current tag in both words has the value, with no
// barrier between the router and the top-k.  (Every CTA writes the next
// layer's logits only after the layer-end barrier, which every reader has
// passed.)  The workspace is zeroed per launch, and tags start at 1.
__device__ __forceinline__ void put_logit(const Cfg &P, int t, int e, double v, unsigned tag) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(v);
    unsigned long long *w = P.logit_ll + 2 * ((size_t)t * P.E + e);
    const unsigned long long w0 = (b & 0xffffffffull) | ((unsigned long long)tag << 32);
    const unsigned long long w1 = (b >> 32) | ((unsigned long long)tag << 32);
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(w), "l"(w0) : "memory");
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(w + 1), "l"(w1) : "memory");
}

// Bounded poll for logit (t, e) of the layer with `tag`; false (error
// recorded) when it does not arrive.
__device__ __forceinline__ bool get_logit(const Cfg &P, int t, int e, unsigned tag, double &v) {
    const unsigned long long *w = P.logit_ll + 2 * ((size_t)t * P.E + e);
    unsigned long long w0, w1;
    unsigned long long t0 = 0;
    for (unsigned it = 0;; ++it) {
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w0) : "l"(w) : "memory");
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w1) : "l"(w + 1) : "memory");
        if ((unsigned)(w0 >> 32) == tag && (unsigned)(w1 >> 32) == tag) break;
        if ((it & 63u) == 63u) {
            if (ldcg_int(P.err) != 0) return false;
            if (t0 == 0) {
                t0 = globaltimer();
            } else if (globaltimer() - t0 > kWaitNs) {
                atomicCAS(P.err, 0, kErrLogits);
                return false;
            }
        }
    }
    v = __longlong_as_double((long long)((w0 & 0xffffffffull) | (w1 << 32)));
    return true;
}

// A consumer warp's wait for ring task `seq`: first until the producer has
// handed the slot to it (the slot's previous task is consumed, so its full
// barrier is in this task's phase), then for the bytes.  Warps take tasks out
// of ring order; without the first wait a warp could test a phase two ahead of
// the barrier's own, which the parity test cannot tell apart.
__device__ __noinline__ bool wait_task(Shared &S, const Cfg &P, unsigned seq) {
    const int s = (int)(seq % (unsigned)P.ns);
    const unsigned ph = (seq / (unsigned)P.ns) & 1u;
    int ok = 1;
    if ((threadIdx.x & 31) == 0 && S.owner[s] != seq) {
        const unsigned long long t0 = globaltimer();
        for (unsigned it = 0; S.owner[s] != seq; ++it) {
            if ((it & 63u) == 63u) {
                if (ldcg_int(P.err) != 0 || globaltimer() - t0 > kWaitNs) {
                    atomicCAS(P.err, 0, kErrOwner);
                    ok = 0;
                    break;
                }
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    // each lane waits for the bytes itself (its own acquire of the copies); the verdict is the warp's
    const int got = ok && mbar_wait(&S.full[s], ph, P.err, kErrFull);
    return __all_sync(0xffffffffu, got) != 0;
}

// Wait of a whole warp for static-region task i of layer l (router rows: 0,
// shared units: 1 + u); the verdict is the warp's.
__device__ __noinline__ bool wait_a(Shared &S, const Cfg &P, int i, int l) {
    const int got = mbar_wait(&S.afull[i], (unsigned)l & 1u, P.err, kErrFull);
    return __all_sync(0xffffffffu, got) != 0;
}

// ------------------------------------------------------------------ phases

constexpr int kXStride = 36;  // floats per 32-column chunk of a staged input (padding spreads the banks)

// Sum over the consumer threads, the same in every CTA (fixed order).
__device__ __forceinline__ float consumer_sum(float v, float *red) {
    v = warp_sum(v);
    consumer_sync();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    consumer_sync();
    float s = 0.f;
#pragma unroll 1
    for (int i = 0; i < kCW; ++i) s += red[i];
    return s;
}

// Layer input rows (bf16) from global memory into the h stage.
__device__ __noinline__ void load_h(const Cfg &P, uint16_t *hs, const uint16_t *src) {
    const int n = P.T * P.H / 8;  // 16-byte units
#pragma unroll 1
    for (int i = threadIdx.x; i < n; i += kCThreads)
        reinterpret_cast<uint4 *>(hs)[i] = __ldcg(reinterpret_cast<const uint4 *>(src) + i);
    consumer_sync();
}

// Output of layer lp: m (every row, from global memory), post-norm,
// residual, layer scalar.  Every CTA computes the whole output; CTA c writes
// its slice of 4-column quads to h_out[lp]; chained stacks keep the output in
// the h stage as the next layer's input.
__device__ __noinline__ void finish_layer(const Cfg &P, Shared &S, uint16_t *hs, int lp) {
    const int T = P.T, H = P.H, H4 = H / 4;
    uint16_t *out = P.h_out + (size_t)lp * T * H;
    const int q0 = (int)((long long)H4 * blockIdx.x / gridDim.x), q1 = (int)((long long)H4 * (blockIdx.x + 1) / gridDim.x);
    const float scalar = P.layer_scalar;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float4 mr[3];
        float ss = 0.f;
#pragma unroll
        for (int r = 0; r < 3; ++r) {
            const int i4 = threadIdx.x + r * kCThreads;
            mr[r] = i4 < H4 ? __ldcg(reinterpret_cast<const float4 *>(P.m + (size_t)t * H) + i4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            ss += mr[r].x * mr[r].x + mr[r].y * mr[r].y + mr[r].z * mr[r].z + mr[r].w * mr[r].w;
        }
        ss = consumer_sum(ss, S.red);
        const float inv = P.post_norm ? 1.0f / sqrtf(ss / (float)H + P.eps) : 1.0f;
#pragma unroll
        for (int r = 0; r < 3; ++r) {
            const int i4 = threadIdx.x + r * kCThreads;
            if (i4 < H4) {
                uint2 hv = reinterpret_cast<const uint2 *>(hs + (size_t)t * H)[i4];
                const float mv[4] = {mr[r].x, mr[r].y, mr[r].z, mr[r].w};
                const uint32_t hw[2] = {hv.x, hv.y};
                uint32_t o[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float hp = bf16_bits_to_float((hw[c >> 1] >> (16 * (c & 1))) & 0xffffu);
                    o[c] = f32_to_bf16_bits_alu((hp + mv[c] * inv) * scalar);
                }
                const uint2 ov = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
                if (i4 >= q0 && i4 < q1) reinterpret_cast<uint2 *>(out + (size_t)t * H)[i4] = ov;
                if (P.chained) reinterpret_cast<uint2 *>(hs + (size_t)t * H)[i4] = ov;
            }
        }
    }
    consumer_sync();
}

// RMS of the layer input, xe = bf16(rmsnorm_no_scale(h)) pre-scaled for the
// code decode into x ([T][CH][kXStride]), and the chunk sums of xe into xs.
__device__ __noinline__ void stage_x(const Cfg &P, Shared &S, const uint16_t *hs, float *x, float *xs) {
    const int T = P.T, H = P.H, H4 = H / 4, CH = P.CH, lane = threadIdx.x & 31;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float ss = 0.f;
#pragma unroll 1
        for (int i = threadIdx.x; i < H / 2; i += kCThreads) {
            const uint32_t v = reinterpret_cast<const uint32_t *>(hs + (size_t)t * H)[i];
            const float a = bf16_bits_to_float(v & 0xffffu), b = bf16_bits_to_float(v >> 16);
            ss = fmaf(a, a, fmaf(b, b, ss));
        }
        ss = consumer_sum(ss, S.red);
        if (threadIdx.x == 0) {
            S.rms[t] = sqrtf(ss / (float)H + P.eps);
            S.rinv[t] = 1.0f / S.rms[t];
        }
    }
    consumer_sync();
    const int n4 = T * H4, rounds = (n4 + kCThreads - 1) / kCThreads;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {  // every consumer runs every round: the shuffles need whole warps
        const int i = r * kCThreads + threadIdx.x;
        float sx = 0.f;
        if (i < n4) {
            const int t = i / H4, col = 4 * (i - t * H4);
            const uint2 hv = reinterpret_cast<const uint2 *>(hs)[i];
            const float ri = S.rinv[t];
            const float x0 = bf16_bits_to_float(f32_to_bf16_bits_alu(bf16_bits_to_float(hv.x & 0xffffu) * ri));
            const float x1 = bf16_bits_to_float(f32_to_bf16_bits_alu(bf16_bits_to_float(hv.x >> 16) * ri));
            const float x2 = bf16_bits_to_float(f32_to_bf16_bits_alu(bf16_bits_to_float(hv.y & 0xffffu) * ri));
            const float x3 = bf16_bits_to_float(f32_to_bf16_bits_alu(bf16_bits_to_float(hv.y >> 16) * ri));
            const int c = col & 7;  // 0 or 4
            float4 v;
            v.x = x0 * code_prescale(c);
            v.y = x1 * code_prescale(c + 1);
            v.z = x2 * code_prescale(c + 2);
            v.w = x3 * code_prescale(c + 3);
            *reinterpret_cast<float4 *>(x + ((size_t)t * CH + (col >> 5)) * kXStride + (col & 31)) = v;
            sx = (x0 + x1) + (x2 + x3);
        }
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        sx += __shfl_xor_sync(0xffffffffu, sx, 4);
        if (i < n4 && (lane & 7) == 0) xs[i >> 3] = sx;  // 8 quads = one chunk: index t * CH + chunk
    }
    consumer_sync();
}

// Router rows [e0, e1) of this CTA and the byte layout of their copy in a ring slot:
// [router_scale: 2H][rows: nrows * H][scale superset: sbb][bias superset: sbb].
struct RouterCopy {
    int e0, nrows;
    unsigned sb_lo, sbb;
};

__device__ __forceinline__ RouterCopy router_copy(const Cfg &P) {
    RouterCopy r;
    const int G = P.GH;
    r.e0 = (int)((long long)P.E * blockIdx.x / gridDim.x);
    const int e1 = (int)((long long)P.E * (blockIdx.x + 1) / gridDim.x);
    r.nrows = e1 - r.e0;
    r.sb_lo = (unsigned)((size_t)r.e0 * G * 2) & ~15u;
    const unsigned sb_hi = ((unsigned)((size_t)e1 * G * 2) + 15u) & ~15u;
    r.sbb = r.nrows > 0 ? sb_hi - r.sb_lo : 0u;
    return r;
}

// R: logits of this CTA's experts for every token.  The dot products run in
// fp64 (h * router_scale is exact in fp32; the 8-bit code becomes a double by
// the 2^52 exponent trick), and the common factor 1 / (rms * sqrt(H)) of a
// token's logits is applied last (it cannot change their order).
__device__ __noinline__ void router_compute(const Cfg &P, Shared &S, const unsigned char *slot, const uint16_t *hs,
                                            double *rpart, bool got, unsigned tag) {
    const int T = P.T, H = P.H, G = P.GH, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const RouterCopy rc = router_copy(P);
    const int items = rc.nrows * T;
    if (items > 0) {
        // the K-split is the one of the CTAs with the most rows, in every CTA: a logit's summation order
        // then does not depend on which CTA computes it, so experts with equal router rows get equal
        // logits (and the tie rule decides between them, as in the per-layer router)
        const int maxi = (P.E + (int)gridDim.x - 1) / (int)gridDim.x * T;
        const int parts = maxi >= kCW ? 1 : kCW / maxi, units = items * parts, nch = H / 16;
        const uint16_t *rsc = reinterpret_cast<const uint16_t *>(slot);
        const unsigned char *rows = slot + 2 * H;
        const int sb_skip = (int)((size_t)rc.e0 * G * 2) - (int)rc.sb_lo;
        const uint16_t *scs = reinterpret_cast<const uint16_t *>(rows + (size_t)rc.nrows * H + sb_skip);
        const uint16_t *bis = reinterpret_cast<const uint16_t *>(rows + (size_t)rc.nrows * H + rc.sbb + sb_skip);
        const double sqrt_h = sqrt((double)H);
#pragma unroll 1
        for (int u = got ? wid : units; u < units; u += kCW) {
            const int item = u / parts, part = u - item * parts;
            const int er = item / T, t = item - er * T;
            const int c0 = nch * part / parts, c1 = nch * (part + 1) / parts;
            const uint16_t *h = hs + (size_t)t * H;
            double acc = 0.0;
#pragma unroll 1
            for (int c = c0 + lane; c < c1; c += 32) {
                const uint4 q = reinterpret_cast<const uint4 *>(rows + (size_t)er * H)[c];
                const uint32_t words[4] = {q.x, q.y, q.z, q.w};
                // the chunk's 16 inputs and scales as 16-byte loads (bf16 pairs)
                const uint4 ha = reinterpret_cast<const uint4 *>(h)[2 * c], hb = reinterpret_cast<const uint4 *>(h)[2 * c + 1];
                const uint4 ra = reinterpret_cast<const uint4 *>(rsc)[2 * c], rb = reinterpret_cast<const uint4 *>(rsc)[2 * c + 1];
                const uint32_t hw[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
                const uint32_t rw[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
                double dots[4] = {0.0, 0.0, 0.0, 0.0}, zss[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                    for (int bi = 0; bi < 4; ++bi) {
                        const int i = wi * 4 + bi;  // element of the chunk
                        const uint32_t hbits = (hw[i >> 1] >> (16 * (i & 1))) & 0xffffu;
                        const uint32_t rbits = (rw[i >> 1] >> (16 * (i & 1))) & 0xffffu;
                        const double z = (double)(bf16_bits_to_float(hbits) * bf16_bits_to_float(rbits));
                        const double qd =
                            __hiloint2double(0x43300000, (int)((words[wi] >> (8 * bi)) & 0xffu)) - 4503599627370496.0;
                        dots[bi] = fma(qd, z, dots[bi]);
                        zss[bi] += z;
                    }
                }
                const double dot = (dots[0] + dots[1]) + (dots[2] + dots[3]);
                const double zs = (zss[0] + zss[1]) + (zss[2] + zss[3]);
                const int g = c >> 2;
                acc += (double)bf16_bits_to_float(scs[er * G + g]) * dot + (double)bf16_bits_to_float(bis[er * G + g]) * zs;
            }
            acc = warp_sum(acc);
            if (lane == 0) {
                if (parts == 1)
                    put_logit(P, t, rc.e0 + er, acc / ((double)S.rms[t] * sqrt_h), tag);
                else
                    rpart[u] = acc;
            }
        }
        if (parts > 1) {
            consumer_sync();  // every consumer, whatever its wait gave
#pragma unroll 1
            for (int item = got ? (int)threadIdx.x : items; item < items; item += kCThreads) {
                double a = 0.0;
                for (int p = 0; p < parts; ++p) a += rpart[item * parts + p];  // fixed order
                const int er = item / T, t = item - er * T;
                put_logit(P, t, rc.e0 + er, a / ((double)S.rms[t] * sqrt_h), tag);
            }
        }
    }
}

// One row of a gate/up unit (slot layout: gate codes [CH][8 rows][16 B] with
// the 128-byte swizzle at 0, up codes at gcb, gate (scale, bias) words
// [GH][8 rows] at 2 gcb, up words after them) against the n <= NT tokens
// toks[]: lanes are 32-column chunks.  g[tt], u[tt]: full sums in every lane.
template <int NT>
__device__ __forceinline__ void g_piece(const Cfg &P, const unsigned char *slot, int row, int n, const int (&tk)[NT],
                                        const float *x, const float *xs, float (&g)[NT], float (&u)[NT]) {
    const int lane = threadIdx.x & 31, CH = P.CH, gcb = P.gcb;
    const unsigned char *sbb = slot + 2 * gcb;
    const int sbs = P.sbs;
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) g[tt] = u[tt] = 0.f;
#pragma unroll 1
    for (int c = lane; c < CH; c += 32) {
        const int sw = (row ^ (c & 7)) << 4;
        // gate and up rows of the chunk against one read of the inputs
        const uint4 qg = *reinterpret_cast<const uint4 *>(slot + c * 128 + sw);
        const uint4 qu = *reinterpret_cast<const uint4 *>(slot + gcb + c * 128 + sw);
        const uint32_t sbg = *reinterpret_cast<const uint32_t *>(sbb + (c >> 1) * 32 + row * 4);
        const uint32_t sbu = *reinterpret_cast<const uint32_t *>(sbb + sbs + (c >> 1) * 32 + row * 4);
        const uint32_t wg[4] = {qg.x, qg.y, qg.z, qg.w}, wu[4] = {qu.x, qu.y, qu.z, qu.w};
        float2 g0[NT], g1[NT], u0[NT], u1[NT];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) g0[tt] = g1[tt] = u0[tt] = u1[tt] = make_float2(0.f, 0.f);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const Decoded8 dg = decode_word(wg[wi]), du = decode_word(wu[wi]);
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                if (tt < n) {
                    const float4 *xp =
                        reinterpret_cast<const float4 *>(x + ((size_t)tk[tt] * CH + c) * kXStride + wi * 8);
                    const float4 xa = xp[0], xb = xp[1];
                    g0[tt] = ffma2(make_float2(dg.f[0], dg.f[1]), make_float2(xa.x, xa.y), g0[tt]);
                    g1[tt] = ffma2(make_float2(dg.f[2], dg.f[3]), make_float2(xa.z, xa.w), g1[tt]);
                    g0[tt] = ffma2(make_float2(dg.f[4], dg.f[5]), make_float2(xb.x, xb.y), g0[tt]);
                    g1[tt] = ffma2(make_float2(dg.f[6], dg.f[7]), make_float2(xb.z, xb.w), g1[tt]);
                    u0[tt] = ffma2(make_float2(du.f[0], du.f[1]), make_float2(xa.x, xa.y), u0[tt]);
                    u1[tt] = ffma2(make_float2(du.f[2], du.f[3]), make_float2(xa.z, xa.w), u1[tt]);
                    u0[tt] = ffma2(make_float2(du.f[4], du.f[5]), make_float2(xb.x, xb.y), u0[tt]);
                    u1[tt] = ffma2(make_float2(du.f[6], du.f[7]), make_float2(xb.z, xb.w), u1[tt]);
                }
            }
        }
        const float s_g = bf16_bits_to_float(sbg & 0xffffu) * kCodeUnscale, b_g = bf16_bits_to_float(sbg >> 16);
        const float s_u = bf16_bits_to_float(sbu & 0xffffu) * kCodeUnscale, b_u = bf16_bits_to_float(sbu >> 16);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
            if (tt < n) {
                const float xsum = xs[tk[tt] * CH + c];
                g[tt] = fmaf(s_g, (g0[tt].x + g0[tt].y) + (g1[tt].x + g1[tt].y), fmaf(b_g, xsum, g[tt]));
                u[tt] = fmaf(s_u, (u0[tt].x + u0[tt].y) + (u1[tt].x + u1[tt].y), fmaf(b_u, xsum, u[tt]));
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
        g[tt] = warp_sum(g[tt]);
        u[tt] = warp_sum(u[tt]);
    }
}

// One 8-row block of a down slot (codes [pc][8 rows][16 B], 128-byte swizzle;
// words [pc/2][8 rows]) against the n <= NT staged inputs apre ([n][pc][kXStride],
// pre-scaled) with chunk sums asum ([n][pc]): lanes are (row r = lane % 8,
// chunk offset j = lane / 8), four chunks per step.  y[tt]: row r's sums in
// lanes r (= lanes 0..7).
template <int NT>
__device__ __forceinline__ void d_block(const unsigned char *codes, const unsigned char *sbp, const float *apre,
                                        const float *asum, int pc, int pcv, int n, float (&y)[NT]) {
    const int lane = threadIdx.x & 31, r = lane & 7, j = lane >> 3;
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) y[tt] = 0.f;
#pragma unroll 1
    for (int c = j; c < pcv; c += 4) {
        const uint4 q = *reinterpret_cast<const uint4 *>(codes + c * 128 + ((r ^ (c & 7)) << 4));
        const uint32_t sbw = *reinterpret_cast<const uint32_t *>(sbp + (c >> 1) * 32 + r * 4);
        const float s = bf16_bits_to_float(sbw & 0xffffu) * kCodeUnscale, b = bf16_bits_to_float(sbw >> 16);
        const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
        float2 a0[NT], a1[NT];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) a0[tt] = a1[tt] = make_float2(0.f, 0.f);
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const Decoded8 d = decode_word(wv[wi]);
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                if (tt < n) {
                    const float4 *xp = reinterpret_cast<const float4 *>(apre + ((size_t)tt * pc + c) * kXStride + wi * 8);
                    const float4 xa = xp[0], xb = xp[1];
                    a0[tt] = ffma2(make_float2(d.f[0], d.f[1]), make_float2(xa.x, xa.y), a0[tt]);
                    a1[tt] = ffma2(make_float2(d.f[2], d.f[3]), make_float2(xa.z, xa.w), a1[tt]);
                    a0[tt] = ffma2(make_float2(d.f[4], d.f[5]), make_float2(xb.x, xb.y), a0[tt]);
                    a1[tt] = ffma2(make_float2(d.f[6], d.f[7]), make_float2(xb.z, xb.w), a1[tt]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
            if (tt < n) {
                const float dsum = (a0[tt].x + a0[tt].y) + (a1[tt].x + a1[tt].y);
                y[tt] = fmaf(s, dsum, fmaf(b, asum[tt * pc + c], y[tt]));
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
        y[tt] += __shfl_xor_sync(0xffffffffu, y[tt], 8);
        y[tt] += __shfl_xor_sync(0xffffffffu, y[tt], 16);
    }
}

// ------------------------------------------------------------------ tensor-core (mma.sync) variants
//
// For batches of 2 to 8 tokens the per-token FMA work of the CUDA-core decode
// grows with T while the bytes do not; these variants use the warp-level
// tensor-core MMA (m16n8k16, BF16 operands, FP32 accumulation), whose N = 8
// columns hold up to 8 tokens at no extra cost.  Codes become exact BF16
// values 128 + q with one mask-or per pair (0x4300 | q is 128 + q), so every
// product is exact; per 64-column group the sum is rescaled:
//     sum_k (s q_k + b) x_k = s * D + (b - 128 s) * sum_k x_k,   D = sum_k (128 + q_k) x_k.
// K order inside a 32-column chunk: lane t of a quad takes word t of a row's
// 16-byte record (columns 8t..8t+7); its two MMAs take the nibble pairs
// (0,4), (1,5) and (2,6), (3,7).  The activations are staged in the same
// order, so the dot products are unchanged.

constexpr int kMaxPieces = 4;  // K-pieces of a gate/up unit on the MMA path

// BF16 pairs (128 + q_j, 128 + q_{j+4}) of a word's nibble pairs j = 0..3.
__device__ __forceinline__ void code_pairs(uint32_t w, uint32_t (&p)[4]) {
    constexpr uint32_t kM = 0x000F000Fu, kB = 0x43004300u;
    p[0] = (w & kM) | kB;
    p[1] = ((w >> 4) & kM) | kB;
    p[2] = ((w >> 8) & kM) | kB;
    p[3] = ((w >> 12) & kM) | kB;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bytes of one token's staged input on the MMA path: [CH][4 lanes][8 bf16] plus 16 bytes of padding,
// so that the 8 tokens read by one load instruction fall in different banks
__host__ __device__ __forceinline__ int xb_token_bytes(int CH) { return CH * 64 + 16; }

// xe of every token as BF16 in the MMA order ([T][CH][t][8]: columns 8t + 0,4,1,5,2,6,3,7)
// and its 64-column group sums xg ([T][GH], fp32).
__device__ __noinline__ void stage_x_mma(const Cfg &P, Shared &S, const uint16_t *hs, unsigned char *xb, float *xg) {
    const int T = P.T, H = P.H, CH = P.CH, GH = P.GH, lane = threadIdx.x & 31;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float ss = 0.f;
#pragma unroll 1
        for (int i = threadIdx.x; i < H / 2; i += kCThreads) {
            const uint32_t v = reinterpret_cast<const uint32_t *>(hs + (size_t)t * H)[i];
            const float a = bf16_bits_to_float(v & 0xffffu), b = bf16_bits_to_float(v >> 16);
            ss = fmaf(a, a, fmaf(b, b, ss));
        }
        ss = consumer_sum(ss, S.red);
        if (threadIdx.x == 0) {
            S.rms[t] = sqrtf(ss / (float)H + P.eps);
            S.rinv[t] = 1.0f / S.rms[t];
        }
    }
    consumer_sync();
    // one thread per 8 columns (a word t of a chunk): 4 threads of a quad make a chunk, 8 a group
    const int n8 = T * H / 8, rounds = (n8 + kCThreads - 1) / kCThreads;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
        const int i = r * kCThreads + threadIdx.x;
        float sx = 0.f;
        if (i < n8) {
            const int t = i / (H / 8), col = 8 * (i - t * (H / 8)), c = col >> 5, wq = (col >> 3) & 3;
            const uint4 hv = *reinterpret_cast<const uint4 *>(hs + (size_t)t * H + col);
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
            const float ri = S.rinv[t];
            uint32_t xv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float h = bf16_bits_to_float((hw[j >> 1] >> (16 * (j & 1))) & 0xffffu);
                xv[j] = f32_to_bf16_bits_alu(h * ri);
                sx += bf16_bits_to_float(xv[j]);
            }
            // order 0,4,1,5,2,6,3,7 as four BF16 pairs
            const uint4 o = make_uint4(xv[0] | (xv[4] << 16), xv[1] | (xv[5] << 16), xv[2] | (xv[6] << 16),
                                       xv[3] | (xv[7] << 16));
            *reinterpret_cast<uint4 *>(xb + (size_t)t * xb_token_bytes(CH) + (size_t)c * 64 + wq * 16) = o;
        }
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        sx += __shfl_xor_sync(0xffffffffu, sx, 4);
        if (i < n8 && (lane & 7) == 0) xg[i >> 3] = sx;  // 8 threads = 64 columns: index t * GH + group
    }
    (void)GH;
    consumer_sync();
}

// Chunks [c0, c1) (whole groups) of a gate/up unit against the n <= 8 tokens
// toks[] on the tensor cores: A rows 0..7 the unit's gate rows, 8..15 its up
// rows; B column j token toks[j].  acc (per lane g = lane / 4, t = lane % 4):
// gate row g and up row g, for the tokens of columns 2t and 2t + 1.
__device__ __forceinline__ void g_piece_mma(const Cfg &P, const unsigned char *slot, int c0, int c1, int n,
                                            const int *toks, const unsigned char *xb, const float *xg,
                                            float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3, gcb = P.gcb, GH = P.GH;
    const int my_tok = g < n ? toks[g] : -1;
    const int tok0 = 2 * t < n ? toks[2 * t] : -1, tok1 = 2 * t + 1 < n ? toks[2 * t + 1] : -1;
    const unsigned char *xrow = xb + (size_t)(my_tok < 0 ? 0 : my_tok) * xb_token_bytes(P.CH);
    const unsigned char *sbg = slot + 2 * gcb, *sbu = slot + 2 * gcb + P.sbs;
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = 0.f;
#pragma unroll 1
    for (int c = c0; c < c1; c += 2) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int ch = c + cc;
            const int off = ch * 128 + ((g ^ (ch & 7)) << 4) + 4 * t;
            const uint32_t wg = *reinterpret_cast<const uint32_t *>(slot + off);
            const uint32_t wu = *reinterpret_cast<const uint32_t *>(slot + gcb + off);
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (my_tok >= 0) xv = *reinterpret_cast<const uint4 *>(xrow + ch * 64 + t * 16);
            uint32_t pg[4], pu[4];
            code_pairs(wg, pg);
            code_pairs(wu, pu);
            mma_bf16(d, pg[0], pu[0], pg[1], pu[1], xv.x, xv.y);
            mma_bf16(d, pg[2], pu[2], pg[3], pu[3], xv.z, xv.w);
        }
        const int grp = c >> 1;
        const uint32_t wsg = *reinterpret_cast<const uint32_t *>(sbg + grp * 32 + g * 4);
        const uint32_t wsu = *reinterpret_cast<const uint32_t *>(sbu + grp * 32 + g * 4);
        const float sg = bf16_bits_to_float(wsg & 0xffffu), bg = fmaf(-128.f, sg, bf16_bits_to_float(wsg >> 16));
        const float su = bf16_bits_to_float(wsu & 0xffffu), bu = fmaf(-128.f, su, bf16_bits_to_float(wsu >> 16));
        const float x0 = tok0 >= 0 ? xg[tok0 * GH + grp] : 0.f, x1 = tok1 >= 0 ? xg[tok1 * GH + grp] : 0.f;
        acc[0] = fmaf(sg, d[0], fmaf(bg, x0, acc[0]));
        acc[1] = fmaf(sg, d[1], fmaf(bg, x1, acc[1]));
        acc[2] = fmaf(su, d[2], fmaf(bu, x0, acc[2]));
        acc[3] = fmaf(su, d[3], fmaf(bu, x1, acc[3]));
    }
}

// bytes of one token's staged down input on the MMA path: [pc][4 lanes][16 bf16] (+16 padding)
__host__ __device__ __forceinline__ int ahl_token_bytes(int pc) { return pc * 128 + 16; }

// One 8-row block of a down slot on the tensor cores: A rows 0..7 the high
// BF16 parts of the tokens' inputs (a = hi + lo), rows 8..15 the low parts;
// B the block's 8 rows.  y[0], y[1] (lane g, t): token g, rows 2t and 2t + 1.
__device__ __forceinline__ void d_block_mma(const unsigned char *codes, const unsigned char *sbp,
                                            const unsigned char *ahl, const float *asg, int pc, int pcv, int n,
                                            float (&y)[2]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const bool mine = g < n;
    const unsigned char *arow = ahl + (size_t)(mine ? g : 0) * ahl_token_bytes(pc);
    y[0] = y[1] = 0.f;
#pragma unroll 1
    for (int c = 0; c < pcv; c += 2) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int ch = c + cc;
            const uint32_t w = *reinterpret_cast<const uint32_t *>(codes + ch * 128 + ((g ^ (ch & 7)) << 4) + 4 * t);
            uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0;
            if (mine) {
                a0 = *reinterpret_cast<const uint4 *>(arow + ch * 128 + t * 32);
                a1 = *reinterpret_cast<const uint4 *>(arow + ch * 128 + t * 32 + 16);
            }
            uint32_t pw[4];
            code_pairs(w, pw);
            mma_bf16(d, a0.x, a0.y, a0.z, a0.w, pw[0], pw[1]);
            mma_bf16(d, a1.x, a1.y, a1.z, a1.w, pw[2], pw[3]);
        }
        const int grp = c >> 1;
        const uint2 sw = *reinterpret_cast<const uint2 *>(sbp + grp * 32 + 2 * t * 4);  // rows 2t, 2t + 1
        const float s0 = bf16_bits_to_float(sw.x & 0xffffu), b0 = fmaf(-128.f, s0, bf16_bits_to_float(sw.x >> 16));
        const float s1 = bf16_bits_to_float(sw.y & 0xffffu), b1 = fmaf(-128.f, s1, bf16_bits_to_float(sw.y >> 16));
        const float as = mine ? asg[g * (pc / 2) + grp] : 0.f;
        y[0] = fmaf(s0, d[0] + d[2], fmaf(b0, as, y[0]));
        y[1] = fmaf(s1, d[1] + d[3], fmaf(b1, as, y[1]));
    }
}

// The logit as an order-preserving 64-bit key (larger logit <=> larger key).
__device__ __forceinline__ unsigned long long logit_key(double v) {
    unsigned long long b = (unsigned long long)__double_as_longlong(v);
    if (b == 0x8000000000000000ull) b = 0ull;  // -0 and +0 are the same logit
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double key_logit(unsigned long long k) {
    const unsigned long long b = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double((long long)b);
}

// K: top-k of every token (ties to the lower expert index; ordered by logit
// desc, index asc), gate weights softmax(logits[top-k]) * per_expert_scale
// in fp64, and the bucketing of the T*k pairs by expert (stable by pair id).
// Every CTA computes the same result from the same logits.  Warp t handles
// token t alone, with no block-wide barrier until the bucketing:
//   1. lane j polls the logits of experts j, 32 + j, ... (all of them in
//      flight at once) and keeps them as order-preserving 64-bit keys;
//   2. k rounds of selection: each lane offers its largest remaining key
//      (the lower expert on equal keys), the warp takes the maximum with two
//      32-bit max-reductions (high word, then low word among the lanes that
//      hold the high word) and the lowest expert index among the lanes that
//      hold the maximum with a min-reduction; the winning lane drops it;
//   3. lanes r < k form the softmax weights (one exp per lane);
// then, over the whole block, the buckets by counting over the T*k pairs.
template <int NSL>
__device__ __noinline__ void topk_bucket(const Cfg &P, Shared &S, const uint16_t *pes, unsigned tag) {
    // called by the T token warps only (T * k <= 32 T pairs: one per thread at most); E <= 32 * NSL
    const int T = P.T, E = P.E, k = P.k, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    {
        const int t = wid, nsl = (E + 31) / 32;
        unsigned long long key[NSL];
        // the lane's logits, four groups of 32 experts per batch of loads (one round trip when they are all there)
#pragma unroll
        for (int sb = 0; sb < NSL; sb += 4) {
            if (sb < nsl) {
                unsigned long long w0[4], w1[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = (sb + q) * 32 + lane;
                    w0[q] = w1[q] = 0ull;
                    if (sb + q < nsl && e < E) {
                        const unsigned long long *w = P.logit_ll + 2 * ((size_t)t * E + e);
                        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w0[q]) : "l"(w) : "memory");
                        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w1[q]) : "l"(w + 1) : "memory");
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = (sb + q) * 32 + lane;
                    key[sb + q] = 0ull;  // below every logit's key: never selected while k <= E
                    if (sb + q < nsl && e < E) {
                        double v;
                        if ((unsigned)(w0[q] >> 32) == tag && (unsigned)(w1[q] >> 32) == tag)
                            v = __longlong_as_double((long long)((w0[q] & 0xffffffffull) | (w1[q] << 32)));
                        else if (!get_logit(P, t, e, tag, v))
                            v = 0.0;  // an error is recorded; the layer's result is void
                        key[sb + q] = logit_key(v);
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) key[sb + q] = 0ull;
            }
        }
#pragma unroll 1
        for (int r = 0; r < k; ++r) {
            unsigned long long best = 0ull;
            int bsl = 0;
#pragma unroll
            for (int sl = 0; sl < NSL; ++sl)
                if (key[sl] > best) {  // strict: the lower group (expert) on equal keys
                    best = key[sl];
                    bsl = sl;
                }
            const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(best >> 32));
            const unsigned lo = __reduce_max_sync(0xffffffffu, (unsigned)(best >> 32) == hi ? (unsigned)best : 0u);
            const unsigned long long top = ((unsigned long long)hi << 32) | lo;
            const unsigned e = __reduce_min_sync(0xffffffffu, best == top ? (unsigned)(bsl * 32 + lane) : 0xffffffffu);
            if (lane == (int)(e & 31u)) {
#pragma unroll
                for (int sl = 0; sl < NSL; ++sl)
                    if (sl == bsl) key[sl] = 0ull;
            }
            if (lane == 0) {
                S.idx[t * k + r] = (int)e;
                S.selv[t * k + r] = key_logit(top);
            }
        }
        __syncwarp();
        // softmax over the k selected logits (rank 0 holds the largest), times per_expert_scale
        const double mx = S.selv[t * k];
        double z = 0.0, ex = 0.0;
        for (int r = lane; r < k; r += 32) {
            const double q = exp(S.selv[t * k + r] - mx);
            if (r == lane) ex = q;
            z += q;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        for (int r = lane; r < k; r += 32) {
            const double q = r == lane ? ex : exp(S.selv[t * k + r] - mx);
            S.wts[t * k + r] = (float)(q / z * (double)bf16_bits_to_float(pes[S.idx[t * k + r]]));
        }
    }
    token_warps_sync(T);
    const int n = T * k;
#pragma unroll 1
    for (int p = threadIdx.x; p < n; p += kCThreads) {
        const int t = p / k, e = S.idx[p];
        int less = 0, eqb = 0, cnt = 0;
#pragma unroll 1
        for (int q = 0; q < n; ++q) {
            const int f = S.idx[q];
            less += f < e;
            eqb += (f == e) & (q < p);
            cnt += f == e;
        }
        S.pos_pair[less + eqb] = p;
        S.pos_tok[less + eqb] = t;
        S.first[p] = eqb == 0;
        S.slot_off[p] = less;  // scratch: moved to the slot's entry below
        S.slot_n[p] = cnt;
    }
    token_warps_sync(T);
    int my_slot = -1, my_e = 0, my_off = 0, my_n = 0;
    if (threadIdx.x < n && S.first[threadIdx.x]) {
        const int p = threadIdx.x, e = S.idx[p];
        int slot = 0;
#pragma unroll 1
        for (int q = 0; q < n; ++q) slot += S.first[q] & (S.idx[q] < e);
        my_slot = slot;
        my_e = e;
        my_off = S.slot_off[p];
        my_n = S.slot_n[p];
    }
    token_warps_sync(T);
    if (my_slot >= 0) {
        S.slot_e[my_slot] = my_e;
        S.slot_off[my_slot] = my_off;
        S.slot_n[my_slot] = my_n;
    }
    if (threadIdx.x == 0) {
        int d = 0;
        for (int q = 0; q < n; ++q) d += S.first[q];
        S.D = d;
    }
    token_warps_sync(T);
}

// ------------------------------------------------------------------ work bookkeeping

// CUDA-core path: piece pi (row row0 + pi) of an 8-row gate/up unit is done;
// every lane holds the row's sums g, u for the n tokens.  The outputs
// a = silu(g) * u wait in shared memory (`part`: [8][kMaxT]); lane 0 of the
// warp that completes the unit writes all 8 rows of every token to global
// memory itself and counts the unit done with one release (its own stores,
// so no further fence), then frees the buffer.
constexpr int kFfmaPart = 8 * kMaxT;  // floats of a unit's staging buffer
template <int NT>
__device__ __forceinline__ void piece_done_ffma(float *part, int *cnt, unsigned long long *empty, unsigned *ready,
                                                int pi, int n, const float (&g)[NT], const float (&u)[NT], float *adst,
                                                const int *ip, int lda, int row0) {
    const int lane = threadIdx.x & 31;
    int last = 0;
    if (lane == 0) {
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
            if (tt < n) part[pi * kMaxT + tt] = silu_mul(g[tt], u[tt]);
        __threadfence_block();
        last = atomicAdd(cnt, 1) == 7;
        if (last) {
            *cnt = 0;
            __threadfence_block();
#pragma unroll 1
            for (int tt = 0; tt < n; ++tt) {
                float *dst = adst + (size_t)ip[tt] * lda + row0;
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = part[q * kMaxT + tt];
            }
            red_release_add(ready, 1u);
            mbar_arrive(empty);
        }
    }
    __syncwarp();
}

// A block task of a down group is done: the last of the group's nblk tasks
// frees the ring slot (and its staged input).
__device__ __forceinline__ void block_done(Shared &S, const Cfg &P, unsigned tseq, int nblk) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        const int s = (int)(tseq % (unsigned)P.ns);
        if (atomicAdd(&S.cnt[s], 1) == nblk - 1) {
            S.cnt[s] = 0;
            S.astate[s] = 0;
            mbar_arrive(&S.empty[s]);
        }
    }
}

// The SwiGLU input of a down group, staged once per group in its ring slot:
// the first warp to arrive waits until every gate/up unit of the slot (the
// shared expert, or routed slot j) is counted done across the grid, then
// copies the n token rows of K-part p, pre-scaled for the code decode
// ([n][pc][kXStride]), with their 32-column sums ([n][pc]); the other warps
// of the group wait for it.
__device__ __noinline__ bool stage_a(Shared &S, const Cfg &P, int s, bool shd, int j, int p, int pc, int pcv, int n,
                                     int off, float *apre, float *asum) {
    const int lane = threadIdx.x & 31;
    int mine = 0, ok = 1;
    if (lane == 0) mine = atomicCAS(const_cast<int *>(&S.astate[s]), 0, 1) == 0;
    mine = __shfl_sync(0xffffffffu, mine, 0);
    if (mine) {
        const int ri = shd ? 0 : 1 + j;
        if (lane == 0) ok = wait_count(P, P.ready + ri, S.exp_ready[ri]);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // the other lanes' loads below come after lane 0's acquire
        if (!ok) return false;
        const int K = shd ? P.Is : P.I;
#pragma unroll 1
        for (int tt = 0; tt < n; ++tt) {
            const float *src = shd ? P.a_sh + (size_t)tt * P.Is : P.a_r + (size_t)(off + tt) * P.I;
            for (int c = lane; c < pcv; c += 32) {
                const int col = (p * pc + c) * 32;
                const float4 *s4 = reinterpret_cast<const float4 *>(src + col);
                float *dst = apre + ((size_t)tt * pc + c) * kXStride;
                float sum = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4 v = col + 4 * q < K ? __ldcg(s4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                    sum += (v.x + v.y) + (v.z + v.w);
                    const int c8 = (4 * q) & 7;  // 0 or 4
                    v.x *= code_prescale(c8);
                    v.y *= code_prescale(c8 + 1);
                    v.z *= code_prescale(c8 + 2);
                    v.w *= code_prescale(c8 + 3);
                    reinterpret_cast<float4 *>(dst)[q] = v;
                }
                asum[tt * pc + c] = sum;
            }
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) S.astate[s] = 2;
        return true;
    }
    if (lane == 0) {
        const unsigned long long t0 = globaltimer();
        for (unsigned it = 0; S.astate[s] != 2; ++it) {
            if ((it & 63u) == 63u && (ldcg_int(P.err) != 0 || globaltimer() - t0 > kWaitNs)) {
                atomicCAS(P.err, 0, kErrStage);
                ok = 0;
                break;
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __threadfence_block();
    return ok != 0;
}

// This CTA's 8-row output blocks [b0, b1), its shared-expert units, and its
// rank rk for the routed gate/up units (unit u goes to the CTA of rank u mod
// G): the CTAs with one output block fewer rank first, so the down blocks and
// the gate/up units even out over the grid.
struct CtaWork {
    int b0, nblk, nshg, rk;
};

__device__ __forceinline__ CtaWork cta_work(const Cfg &P) {
    CtaWork w;
    const int G = gridDim.x, c = blockIdx.x;
    w.b0 = (int)((long long)P.nrb8 * c / G);
    w.nblk = (int)((long long)P.nrb8 * (c + 1) / G) - w.b0;
    w.nshg = c < P.units_s ? (P.units_s - 1 - c) / G + 1 : 0;
    const int q = P.nrb8 / G, nhigh = P.nrb8 - q * G;  // CTAs with q + 1 blocks
    const int hb = w.b0 - q * c;                       // of them before this CTA
    w.rk = w.nblk == q ? c - hb : (G - nhigh) + hb;
    return w;
}

// Down group gi of a layer: the shared expert's K-part p (gi < parts_s), or
// routed slot j's K-part p.
struct DGroup {
    bool shd;
    int j, p, pc, dcb, sbd, pcv;
};

__device__ __forceinline__ DGroup dgroup(const Cfg &P, int gi) {
    DGroup d;
    d.shd = gi < P.parts_s;
    if (d.shd) {
        d.j = -1;
        d.p = gi;
    } else {
        d.j = (gi - P.parts_s) / P.parts_r;
        d.p = gi - P.parts_s - d.j * P.parts_r;
    }
    d.pc = d.shd ? P.pc_s : P.pc_r;
    d.dcb = d.shd ? P.dcb_s : P.dcb_r;
    d.sbd = d.shd ? P.sbd_s : P.sbd_r;
    const int CK = (d.shd ? P.Is : P.I) / 32;
    d.pcv = min(d.pc, CK - d.p * d.pc);
    return d;
}

// The MMA path's staging of a down group's input: for each of its n tokens,
// a = hi + lo (two BF16 values, round to nearest each) in the MMA order
// ([n][pc][t][16 bf16] + padding per token) and the 64-column sums of hi + lo
// ([n][pc/2], fp32).  One lane per 32-column chunk; the first warp of the
// group stages, the others wait (as stage_a).
__device__ __noinline__ bool stage_a_mma(Shared &S, const Cfg &P, volatile int *state, bool shd, int j, int p, int pc,
                                         int pcv, int n, int off, unsigned char *ahl, float *asg) {
    const int lane = threadIdx.x & 31;
    int mine = 0, ok = 1;
    if (lane == 0) mine = atomicCAS(const_cast<int *>(state), 0, 1) == 0;
    mine = __shfl_sync(0xffffffffu, mine, 0);
    if (mine) {
        const int ri = shd ? 0 : 1 + j;
        if (lane == 0) ok = wait_count(P, P.ready + ri, S.exp_ready[ri]);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // the other lanes' loads below come after lane 0's acquire
        if (!ok) return false;
        // (token, chunk) pairs over the lanes: pcv is even, so lanes w and w ^ 1 hold the two chunks of a group
#pragma unroll 1
        for (int w0 = 0; w0 < n * pcv; w0 += 32) {
            const int wq = w0 + lane, tt = wq < n * pcv ? wq / pcv : 0, c = wq < n * pcv ? wq - tt * pcv : pcv;
            const float *src = shd ? P.a_sh + (size_t)tt * P.Is : P.a_r + (size_t)(off + tt) * P.I;
            float sum = 0.f;
            if (c < pcv) {
                const float4 *s4 = reinterpret_cast<const float4 *>(src + (p * pc + c) * 32);
                unsigned char *dst = ahl + (size_t)tt * ahl_token_bytes(pc) + c * 128;
#pragma unroll
                for (int w = 0; w < 4; ++w) {  // columns 8w .. 8w + 7 of the chunk
                    const float4 va = __ldcg(s4 + 2 * w), vb = __ldcg(s4 + 2 * w + 1);
                    const float v[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        hi[q] = f32_to_bf16_bits_alu(v[q]);
                        lo[q] = f32_to_bf16_bits_alu(v[q] - bf16_bits_to_float(hi[q]));
                        sum += bf16_bits_to_float(hi[q]) + bf16_bits_to_float(lo[q]);
                    }
                    const uint4 o0 = make_uint4(hi[0] | (hi[4] << 16), lo[0] | (lo[4] << 16), hi[1] | (hi[5] << 16),
                                                lo[1] | (lo[5] << 16));
                    const uint4 o1 = make_uint4(hi[2] | (hi[6] << 16), lo[2] | (lo[6] << 16), hi[3] | (hi[7] << 16),
                                                lo[3] | (lo[7] << 16));
                    reinterpret_cast<uint4 *>(dst + w * 32)[0] = o0;
                    reinterpret_cast<uint4 *>(dst + w * 32)[1] = o1;
                }
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);  // the two chunks of a group
            if (c < pcv && (c & 1) == 0) asg[tt * (pc / 2) + (c >> 1)] = sum;
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) *state = 2;
        return true;
    }
    if (lane == 0) {
        const unsigned long long t0 = globaltimer();
        for (unsigned it = 0; *state != 2; ++it) {
            if ((it & 63u) == 63u && (ldcg_int(P.err) != 0 || globaltimer() - t0 > kWaitNs)) {
                atomicCAS(P.err, 0, kErrStage);
                ok = 0;
                break;
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __threadfence_block();
    return ok != 0;
}

// MMA path: a K-piece of a gate/up unit is done (its partial sums are in
// `part`); true (warp-uniform) for the warp that completes the unit, which
// then owns the slot's partials.
__device__ __forceinline__ bool piece_last(int *cnt, int npc) {
    __syncwarp();
    int last = 0;
    if ((threadIdx.x & 31) == 0) {
        __threadfence_block();
        last = atomicAdd(cnt, 1) == npc - 1;
        if (last) *cnt = 0;
        __threadfence_block();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    return last != 0;
}

// The completing warp of a unit counts it done in global memory (release) and frees its buffer.
__device__ __forceinline__ void unit_release(unsigned long long *empty, unsigned *ready) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        __threadfence();
        red_release_add(ready, 1u);
        mbar_arrive(empty);
    }
}

// MMA path: one K-piece of a gate/up unit (8 rows) for the tokens toks[0..n);
// the warp completing the unit sums the pieces' partials in order and stores
// a = silu(g) * u for its 8 rows (row0 .. row0 + 7 of `a`, token tt of the
// list at a + aidx[tt] * lda).
//   slot: the unit's bytes; part: its partial-sum buffer ([kMaxPieces][128] floats); cnt / empty: its
//   piece counter and the barrier that frees its buffer.
__device__ __forceinline__ void unit_piece_mma(const Cfg &P, const unsigned char *slot, float *part, int *cnt,
                                               unsigned long long *empty, int pi, int npc, int n, const int *toks,
                                               const int *aidx, float *a, int lda, int row0, const unsigned char *xb,
                                               const float *xg, unsigned *ready) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int gpp = (P.GH + npc - 1) / npc;
    const int c0 = min(P.CH, 2 * pi * gpp), c1 = min(P.CH, c0 + 2 * gpp);
    float acc[4];
    g_piece_mma(P, slot, c0, c1, n, toks, xb, xg, acc);
    float *mine = part + (size_t)pi * 128 + lane * 4;
    *reinterpret_cast<float4 *>(mine) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    if (!piece_last(cnt, npc)) return;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < npc; ++q) {  // fixed order
        const float4 v = *reinterpret_cast<const float4 *>(part + (size_t)q * 128 + lane * 4);
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
    }
    if (2 * t < n) a[(size_t)aidx[2 * t] * lda + row0 + g] = silu_mul(sum.x, sum.z);
    if (2 * t + 1 < n) a[(size_t)aidx[2 * t + 1] * lda + row0 + g] = silu_mul(sum.y, sum.w);
    unit_release(empty, ready);
}

// ------------------------------------------------------------------ consumers

template <int NT, bool kMma>
__device__ __noinline__ void consumer_main(const Params &Pk, Shared &S, unsigned char *base) {
    // kMma: the tensor-core (mma.sync) variants; otherwise CUDA-core FMAs for at most NT tokens
    const Cfg &P = S.c;
    const int T = P.T, H = P.H, G = gridDim.x, c = blockIdx.x, ns = P.ns;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    unsigned char *ring = base + P.off_ring;
    const unsigned char *abase = base + P.off_a;            // static region: router rows, shared units
    float *x = reinterpret_cast<float *>(base + P.off_x);   // FFMA path: pre-scaled fp32 xe
    unsigned char *xb = base + P.off_x;                    // MMA path: BF16 xe in the MMA order
    float *xs = reinterpret_cast<float *>(base + P.off_xs); // chunk sums (FFMA) or group sums (MMA)
    uint16_t *hs = reinterpret_cast<uint16_t *>(base + P.off_h);
    float *ybuf = reinterpret_cast<float *>(base + P.off_y);
    float *part = reinterpret_cast<float *>(base + P.off_part);
    const CtaWork cw = cta_work(P);
    unsigned seq = 0, nbar = 0;
    bool ok = true;
#pragma unroll 1
    for (int l = 0; l < P.L && ok; ++l) {
        // ---------------------------------------------------------- F: the layer's input
        if (l == 0) {
            load_h(P, hs, P.h_in);
        } else {
            if (!(ok = grid_wait(P, S, ++nbar))) break;  // every CTA has written m of layer l-1
            finish_layer(P, S, hs, l - 1);
            if (!P.chained) load_h(P, hs, P.h_in + (size_t)l * T * H);
        }
        if (kMma)
            stage_x_mma(P, S, hs, xb, xs);
        else
            stage_x(P, S, hs, x, xs);
        // ---------------------------------------------------------- R: router rows of this CTA
        {
            const bool got = wait_a(S, P, 0, l);
            router_compute(P, S, abase, hs, S.rpart, got, (unsigned)l + 1u);
            consumer_sync();
            if (threadIdx.x == 0) mbar_arrive(&S.aempty);
        }
        // ---------------------------------------------------------- K (token warps) and S (the others)
        // The T token warps rank the logits (they carry the layer's tag: no barrier before reading them)
        // and publish the routing tables; meanwhile the other warps run the shared units already in the
        // static region, which need only xe.
        const int nss = min(cw.nshg, P.ua);
        if (wid < T) {
            if (P.E <= 128)
                topk_bucket<4>(P, S, Pk.layers[l].per_expert_scale, (unsigned)l + 1u);
            else if (P.E <= 256)
                topk_bucket<8>(P, S, Pk.layers[l].per_expert_scale, (unsigned)l + 1u);
            else
                topk_bucket<kMaxSl>(P, S, Pk.layers[l].per_expert_scale, (unsigned)l + 1u);
            if (threadIdx.x == 0) {
                const int good = ldcg_int(P.err) == 0;
                S.kverdict = good;
                if (good) {
                    S.exp_ready[0] += (unsigned)P.units_s;
                    for (int j = 0; j < S.D; ++j) S.exp_ready[1 + j] += (unsigned)P.units_r;
                }
                if (P.xm)
                    for (int i = 0; i < kMaxStage; ++i) S.xstate[i] = 0;  // this layer's experts are not staged yet
                __threadfence_block();
                S.tables_layer = l + 1;  // the producer and the other warps may go on
            }
        } else {
            const int nsw = kCW - T;  // warps on the shared units
            const int npc = kMma ? min(kMaxPieces, max(1, (nsw + max(nss, 1) - 1) / max(nss, 1))) : 8;
#pragma unroll 1
            for (int i = wid - T; i < nss * npc; i += nsw) {
                const int ui = i / npc, pi = i - ui * npc;
                if (!wait_a(S, P, 1 + ui, l)) break;
                const unsigned char *unit = abase + P.a_rbytes + (size_t)ui * P.a_ubytes;
                const int row0 = (c + ui * G) * 8;  // first row of the unit in the shared gate/up matrices
                if (kMma) {
                    unit_piece_mma(P, unit, part + (size_t)(ns + ui) * kMaxPieces * 128, &S.acnt[1 + ui], &S.aempty,
                                   pi, npc, T, S.toks_sh, S.toks_sh, P.a_sh, P.Is, row0, xb, xs, P.ready);
                } else {
                    int tk[NT];
#pragma unroll
                    for (int tt = 0; tt < NT; ++tt) tk[tt] = tt < T ? tt : 0;
                    float g[NT], u[NT];
                    g_piece<NT>(P, unit, pi, T, tk, x, xs, g, u);
                    piece_done_ffma<NT>(part + (size_t)(ns + ui) * kFfmaPart, &S.acnt[1 + ui], &S.aempty, P.ready, pi,
                                        T, g, u, P.a_sh, S.toks_sh, P.Is, row0);
                }
            }
        }
        // every warp: this layer's routing tables (bounded wait), then the ring items
        {
            int seen = 1;
            if (lane == 0) {
                const unsigned long long t0 = globaltimer();
                for (unsigned it = 0; S.tables_layer < l + 1; ++it)
                    if ((it & 63u) == 63u && (ldcg_int(P.err) != 0 || globaltimer() - t0 > kWaitNs)) {
                        atomicCAS(P.err, 0, kErrTables);
                        seen = 0;
                        break;
                    }
                __threadfence_block();
            }
            seen = __shfl_sync(0xffffffffu, seen, 0);
            if (!(ok = seen && S.kverdict != 0)) break;
        }
        // ---------------------------------------------------------- G and D
        // the gate/up units of the ring (routed, then shared ones that did not fit the static region),
        // then the down blocks
        const int D = S.D, nu = D * P.units_r;
        const int nrg = cw.rk < nu ? (nu - 1 - cw.rk) / G + 1 : 0;
        // down groups by output rows: the shared expert's, and (unless the routed down work goes by
        // expert) every routed slot's
        const int ngr = cw.nblk > 0 ? P.parts_s + ((kMma && P.xm) ? 0 : D * P.parts_r) : 0;
        const int ngu = nrg + (cw.nshg - nss);  // ring gate/up units: routed, shared
        // expert-major routed down items [xg0, xg1) of the grid's D * ipe (expert, 32-row block) items
        const int xtot = (kMma && P.xm) ? D * P.ipe : 0;
        const int xg0 = kMma ? (int)((long long)xtot * c / G) : 0, xg1 = kMma ? (int)((long long)xtot * (c + 1) / G) : 0;
        const int nxm = xg1 - xg0, xj0 = kMma && nxm > 0 ? xg0 / P.ipe : 0;
        // K-pieces per ring unit: enough for every warp while at most ns units are resident at once
        const int nres = max(1, min(ngu, ns));
        const int npc = kMma ? min(kMaxPieces, (kCW + nres - 1) / nres) : 8;
        const int nitems = ngu * npc + ngr * cw.nblk + nxm * kXmBlk;
#pragma unroll 1
        for (int i = wid; i < nitems; i += kCW) {
            if (i < ngu * npc) {
                const int ui = i / npc, pi = i - ui * npc;
                const unsigned tseq = seq + (unsigned)ui;
                if (!wait_task(S, P, tseq)) break;
                int n, row0, lda;
                const int *tp, *ip;
                float *adst;
                unsigned *rdy;
                if (ui < nrg) {  // routed unit: slot j's rows sub*8 .. sub*8+7
                    const int u = cw.rk + ui * G, j = u / P.units_r, sub = u - j * P.units_r, off = S.slot_off[j];
                    n = S.slot_n[j];
                    tp = S.pos_tok + off;
                    ip = S.pos_idx + off;
                    adst = P.a_r;
                    lda = P.I;
                    row0 = sub * 8;
                    rdy = P.ready + 1 + j;
                } else {  // shared unit that did not fit the static region
                    n = T;
                    tp = ip = S.toks_sh;
                    adst = P.a_sh;
                    lda = P.Is;
                    row0 = (c + (nss + ui - nrg) * G) * 8;
                    rdy = P.ready;
                }
                const int s = (int)(tseq % (unsigned)ns);
                if (kMma) {
                    unit_piece_mma(P, ring + (size_t)s * P.slot_bytes, part + (size_t)s * kMaxPieces * 128, &S.cnt[s],
                                   &S.empty[s], pi, npc, n, tp, ip, adst, lda, row0, xb, xs, rdy);
                } else {
                    int tk[NT];
#pragma unroll
                    for (int tt = 0; tt < NT; ++tt) tk[tt] = tp[tt < n ? tt : 0];
                    float g[NT], uu[NT];
                    g_piece<NT>(P, ring + (size_t)s * P.slot_bytes, pi, n, tk, x, xs, g, uu);
                    piece_done_ffma<NT>(part + (size_t)s * kFfmaPart, &S.cnt[s], &S.empty[s], rdy, pi, n, g, uu, adst,
                                        ip, lda, row0);
                }
            } else if (kMma && i >= ngu * npc + ngr * cw.nblk) {
                // expert-major routed down: item xi (expert j, 32-row block q), block bi of it, against the
                // expert's input staged once in this CTA
                const int xi = (i - ngu * npc - ngr * cw.nblk) / kXmBlk, bi = (i - ngu * npc - ngr * cw.nblk) % kXmBlk;
                const int g = xg0 + xi, j = g / P.ipe, q = g - j * P.ipe;
                const unsigned tseq = seq + (unsigned)(ngu + ngr + xi);
                if (!wait_task(S, P, tseq)) break;
                const int n = S.slot_n[j], off = S.slot_off[j], si = j - xj0;
                if (si >= P.nstage) {  // the plan bounds the experts per CTA; never expected
                    if (lane == 0) atomicCAS(P.err, 0, kErrStage);
                    break;
                }
                unsigned char *area = base + P.off_stage + (size_t)si * P.stage_bytes;
                float *asg = reinterpret_cast<float *>(area + (size_t)n * ahl_token_bytes(P.pc_r));
                if (!stage_a_mma(S, P, &S.xstate[si], false, j, 0, P.pc_r, P.pc_r, n, off, area, asg)) break;
                const int s = (int)(tseq % (unsigned)ns);
                const unsigned char *slot = ring + (size_t)s * P.slot_bytes;
                float y[2];
                d_block_mma(slot + bi * P.dcb_r, slot + kXmBlk * P.dcb_r + bi * P.sbd_r, area, asg, P.pc_r, P.pc_r, n,
                            y);
                const int g8 = lane >> 2, t4 = lane & 3;
                if (g8 < n) {
                    float *dst = P.y_r + (size_t)S.pos_pair[off + g8] * H + (q * kXmBlk + bi) * 8 + 2 * t4;
                    *reinterpret_cast<float2 *>(dst) = make_float2(y[0], y[1]);
                }
                block_done(S, P, tseq, kXmBlk);
            } else {
                const int di = i - ngu * npc, gi = di / cw.nblk, bi = di - gi * cw.nblk;
                const unsigned tseq = seq + (unsigned)(ngu + gi);
                if (!wait_task(S, P, tseq)) break;
                const DGroup dg = dgroup(P, gi);
                const int n = dg.shd ? T : S.slot_n[dg.j], off = dg.shd ? 0 : S.slot_off[dg.j];
                const int s = (int)(tseq % (unsigned)ns);
                unsigned char *slot = ring + (size_t)s * P.slot_bytes;
                unsigned char *area = slot + cw.nblk * (dg.dcb + dg.sbd);
                const unsigned char *codes = slot + bi * dg.dcb, *sbp = slot + cw.nblk * dg.dcb + bi * dg.sbd;
                if (kMma) {
                    float *asg = reinterpret_cast<float *>(area + (size_t)n * ahl_token_bytes(dg.pc));
                    if (!stage_a_mma(S, P, &S.astate[s], dg.shd, dg.j, dg.p, dg.pc, dg.pcv, n, off, area, asg)) break;
                    float y[2];
                    d_block_mma(codes, sbp, area, asg, dg.pc, dg.pcv, n, y);
                    const int g8 = lane >> 2, t4 = lane & 3;
                    if (g8 < n) {
                        // by expert, the routed outputs go to global memory and ybuf keeps the shared ones only
                        const int entry = dg.shd ? (P.xm ? 0 : T * P.k * P.parts_r) + dg.p * T + g8
                                                 : S.pos_pair[off + g8] * P.parts_r + dg.p;
                        ybuf[(size_t)entry * P.yrows + bi * 8 + 2 * t4] = y[0];
                        ybuf[(size_t)entry * P.yrows + bi * 8 + 2 * t4 + 1] = y[1];
                    }
                } else {
                    float *apre = reinterpret_cast<float *>(area);
                    float *asum = apre + (size_t)n * dg.pc * kXStride;
                    if (!stage_a(S, P, s, dg.shd, dg.j, dg.p, dg.pc, dg.pcv, n, off, apre, asum)) break;
                    float y[NT];
                    d_block<NT>(codes, sbp, apre, asum, dg.pc, dg.pcv, n, y);
                    if (lane < 8) {
                        const int row = bi * 8 + lane;
#pragma unroll
                        for (int tt = 0; tt < NT; ++tt) {
                            if (tt < n) {
                                const int entry = dg.shd ? T * P.k * P.parts_r + dg.p * T + tt
                                                         : S.pos_pair[off + tt] * P.parts_r + dg.p;
                                ybuf[(size_t)entry * P.yrows + row] = y[tt];
                            }
                        }
                    }
                }
                block_done(S, P, tseq, cw.nblk);
            }
        }
        seq += (unsigned)(ngu + ngr + nxm);
        consumer_sync();
        if (kMma && P.xm) {  // every CTA's routed outputs are written before any CTA sums its rows
            if (!ok) break;
            if (threadIdx.x == 0) grid_arrive(P);
            if (!(ok = grid_wait(P, S, ++nbar))) break;
        }
        // ---------------------------------------------------------- the combine of this CTA's rows
        if (cw.nblk > 0) {
            const int nrows = cw.nblk * 8, r0 = cw.b0 * 8, k = P.k, pr = P.parts_r;
#pragma unroll 1
            for (int i = threadIdx.x; i < T * nrows; i += kCThreads) {
                const int t = i / nrows, r = i - t * nrows;
                float acc = 0.f;
#pragma unroll 1
                for (int s2 = 0; s2 < k; ++s2) {
                    float ys = 0.f;
                    if (kMma && P.xm)  // written by the CTAs that own the expert's rows (before the barrier above)
                        ys = __ldcg(P.y_r + (size_t)(t * k + s2) * H + r0 + r);
                    else
                        for (int p = 0; p < pr; ++p) ys += ybuf[(size_t)((t * k + s2) * pr + p) * P.yrows + r];
                    acc = fmaf(S.wts[t * k + s2], ys, acc);
                }
                float sh = 0.f;
                const int sh0 = (kMma && P.xm) ? 0 : T * k * pr;
                for (int p = 0; p < P.parts_s; ++p) sh += ybuf[(size_t)(sh0 + p * T + t) * P.yrows + r];
                P.m[(size_t)t * H + r0 + r] = acc + sh;
            }
        }
        consumer_sync();
        if (threadIdx.x == 0) grid_arrive(P);  // m rows written
    }
    if (ok && grid_wait(P, S, ++nbar)) finish_layer(P, S, hs, P.L - 1);
}

// ------------------------------------------------------------------ producer

// Hand ring slot of task `sq` to the task and arm its full barrier for
// `bytes`; null on a timeout or a recorded error.
__device__ __forceinline__ unsigned char *claim(Shared &S, const Cfg &P, unsigned char *ring, unsigned sq,
                                               unsigned bytes) {
    const int s = (int)(sq % (unsigned)P.ns);
    const unsigned q = sq / (unsigned)P.ns;
    if (q > 0 && !mbar_wait(&S.empty[s], (q - 1u) & 1u, P.err, kErrEmpty)) return nullptr;
    S.owner[s] = sq;
    mbar_expect_tx(&S.full[s], bytes);
    return ring + (size_t)s * P.slot_bytes;
}

// The static part of layer l -- the router rows of this CTA and its shared
// gate/up units, which do not depend on the routing -- into the static
// region, once the previous layer's copy there is consumed.
__device__ __noinline__ bool issue_seg_a(Shared &S, const Cfg &P, const moe_layer_w &W, const CUtensorMap *mp,
                                         unsigned char *abase, const CtaWork &cw, int l) {
    const int H = P.H, G = gridDim.x, c = blockIdx.x;
    if (l > 0 && !mbar_wait(&S.aempty, (unsigned)(l - 1) & 1u, P.err, kErrEmpty)) return false;
    {
        const RouterCopy rc = router_copy(P);
        const unsigned rows_bytes = (unsigned)rc.nrows * H;
        unsigned long long *fb = &S.afull[0];
        mbar_expect_tx(fb, 2u * H + rows_bytes + 2u * rc.sbb);
        bulk_g2s(abase, W.router_scale, 2u * H, fb);
        if (rc.nrows > 0) {
            bulk_g2s(abase + 2 * H, W.router_q + (size_t)rc.e0 * (H / 4), rows_bytes, fb);
            bulk_g2s(abase + 2 * H + rows_bytes, reinterpret_cast<const char *>(W.router_s) + rc.sb_lo, rc.sbb, fb);
            bulk_g2s(abase + 2 * H + rows_bytes + rc.sbb, reinterpret_cast<const char *>(W.router_b) + rc.sb_lo,
                     rc.sbb, fb);
        }
    }
    const unsigned ubytes = 2u * P.CH * 128u + 2u * P.GH * 32u;
#pragma unroll 1
    for (int ui = 0; ui < min(cw.nshg, P.ua); ++ui) {
        const int u = c + ui * G, rb = u >> 2, x = u & 3;
        unsigned char *dst = abase + P.a_rbytes + (size_t)ui * P.a_ubytes;
        unsigned long long *fb = &S.afull[1 + ui];
        mbar_expect_tx(fb, ubytes);
        tma_load_3d(dst, mp + kMapShGateQ, 32 * x, 0, rb, fb);
        tma_load_3d(dst + P.gcb, mp + kMapShUpQ, 32 * x, 0, rb, fb);
        tma_load_3d(dst + 2 * P.gcb, mp + kMapShGateSb, 8 * x, 0, rb, fb);
        tma_load_3d(dst + 2 * P.gcb + P.sbs, mp + kMapShUpSb, 8 * x, 0, rb, fb);
    }
    return true;
}

// Coordinates of routed gate/up unit u (of the grid's D * units_r) of the layer.
__device__ __forceinline__ void routed_unit(const Cfg &P, const Shared &S, int u, int &rb, int &x) {
    const int j = u / P.units_r, sub = u - j * P.units_r;
    rb = S.slot_e[j] * (P.I / 32) + (sub >> 2);
    x = sub & 3;
}

// Row block of 8-row output block b of down group dg (routed: of slot j's expert).
__device__ __forceinline__ int down_rb(const Cfg &P, const Shared &S, const DGroup &dg, int b) {
    return (dg.shd ? 0 : S.slot_e[dg.j] * (P.H / 32)) + (b >> 2);
}

template <bool kMma>
__device__ __noinline__ void producer_main(const Params &Pk, Shared &S, unsigned char *base) {
    if ((threadIdx.x & 31) != 0) return;
    const Cfg &P = S.c;
    const int G = gridDim.x, c = blockIdx.x, ns = P.ns;
    unsigned char *ring = base + P.off_ring;
    unsigned char *abase = base + P.off_a;
    const CtaWork cw = cta_work(P);
    unsigned seq = 0;
    int a_issued = 0;  // layers whose static part has been issued
    for (int i = 0; i < kMaps * min(P.L, 2); ++i) prefetch_map(P.maps + i);
    bool ok = issue_seg_a(S, P, Pk.layers[0], P.maps, abase, cw, 0);
    if (ok) a_issued = 1;
#pragma unroll 1
    for (int l = 0; l < P.L && ok; ++l) {
        if (l + 2 < P.L)
            for (int i = 0; i < kMaps; ++i) prefetch_map(P.maps + (size_t)(l + 2) * kMaps + i);
        {  // this layer's routing tables
            const unsigned long long t0 = globaltimer();
            for (unsigned it = 0; S.tables_layer < l + 1; ++it) {
                if ((it & 63u) == 63u && (ldcg_int(P.err) != 0 || globaltimer() - t0 > kWaitNs)) {
                    atomicCAS(P.err, 0, kErrTables);
                    ok = false;
                    break;
                }
                __nanosleep(64);
            }
            if (!ok) break;
            __threadfence_block();
            if (!S.kverdict) {  // the routing of this layer failed: the consumers stop
                ok = false;
                break;
            }
        }
        const CUtensorMap *mp = P.maps + (size_t)l * kMaps;
        const int D = S.D, nu = D * P.units_r;
        const int nrg = cw.rk < nu ? (nu - 1 - cw.rk) / G + 1 : 0;
        const int ngr = cw.nblk > 0 ? P.parts_s + ((kMma && P.xm) ? 0 : D * P.parts_r) : 0;
        const int xtot = (kMma && P.xm) ? D * P.ipe : 0;
        const int xg0 = kMma ? (int)((long long)xtot * c / G) : 0, xg1 = kMma ? (int)((long long)xtot * (c + 1) / G) : 0;
        // routed gate/up units first (the layer's critical path); once the ring is full, the rest of them
        // are asked into L2 before the loop waits for free slots
        const unsigned ubytes = 2u * P.CH * 128u + 2u * P.GH * 32u;
#pragma unroll 1
        for (int ui = 0; ui < nrg && ok; ++ui) {
            int rb, x;
            if (ui == ns) {
#pragma unroll 1
                for (int uj = ns; uj < nrg; ++uj) {
                    routed_unit(P, S, cw.rk + uj * G, rb, x);
                    tma_prefetch_3d(mp + kMapGateQ, 32 * x, 0, rb);
                    tma_prefetch_3d(mp + kMapUpQ, 32 * x, 0, rb);
                }
            }
            routed_unit(P, S, cw.rk + ui * G, rb, x);
            unsigned char *dst = claim(S, P, ring, seq, ubytes);
            if (!dst) {
                ok = false;
                break;
            }
            unsigned long long *fb = &S.full[seq % (unsigned)ns];
            tma_load_3d(dst, mp + kMapGateQ, 32 * x, 0, rb, fb);
            tma_load_3d(dst + P.gcb, mp + kMapUpQ, 32 * x, 0, rb, fb);
            tma_load_3d(dst + 2 * P.gcb, mp + kMapGateSb, 8 * x, 0, rb, fb);
            tma_load_3d(dst + 2 * P.gcb + P.sbs, mp + kMapUpSb, 8 * x, 0, rb, fb);
            ++seq;
        }
        // shared units that did not fit the static region
#pragma unroll 1
        for (int ui = min(cw.nshg, P.ua); ui < cw.nshg && ok; ++ui) {
            const int u = c + ui * G, rb = u >> 2, x = u & 3;
            unsigned char *dst = claim(S, P, ring, seq, ubytes);
            if (!dst) {
                ok = false;
                break;
            }
            unsigned long long *fb = &S.full[seq % (unsigned)ns];
            tma_load_3d(dst, mp + kMapShGateQ, 32 * x, 0, rb, fb);
            tma_load_3d(dst + P.gcb, mp + kMapShUpQ, 32 * x, 0, rb, fb);
            tma_load_3d(dst + 2 * P.gcb, mp + kMapShGateSb, 8 * x, 0, rb, fb);
            tma_load_3d(dst + 2 * P.gcb + P.sbs, mp + kMapShUpSb, 8 * x, 0, rb, fb);
            ++seq;
        }
        // the next layer's static part: its region was consumed before this layer's top-k
        if (ok && l + 1 < P.L) {
            ok = issue_seg_a(S, P, Pk.layers[l + 1], P.maps + (size_t)(l + 1) * kMaps, abase, cw, l + 1);
            if (ok) a_issued = l + 2;
        }
        // the down groups, in ring order
#pragma unroll 1
        for (int gi = 0; gi < ngr && ok; ++gi) {
            const DGroup dg = dgroup(P, gi);
            const unsigned gbytes = (unsigned)cw.nblk * (unsigned)(dg.pc * 128 + dg.pc * 16);
            unsigned char *dst = claim(S, P, ring, seq, gbytes);
            if (!dst) {
                ok = false;
                break;
            }
            unsigned long long *fb = &S.full[seq % (unsigned)ns];
            for (int bi = 0; bi < cw.nblk; ++bi) {
                const int b = cw.b0 + bi, rb = down_rb(P, S, dg, b);
                tma_load_3d(dst + bi * dg.dcb, mp + (dg.shd ? kMapShDownQ : kMapDownQ), 32 * (b & 3), dg.p * dg.pc, rb,
                            fb);
                tma_load_3d(dst + cw.nblk * dg.dcb + bi * dg.sbd, mp + (dg.shd ? kMapShDownSb : kMapDownSb), 8 * (b & 3),
                            dg.p * (dg.pc / 2), rb, fb);
            }
            ++seq;
        }
        // expert-major routed down items: expert j's kXmBlk 8-row blocks from block q * kXmBlk, in item order
#pragma unroll 1
        for (int g = xg0; g < xg1 && ok; ++g) {
            const int j = g / P.ipe, q = g - j * P.ipe;
            unsigned char *dst = claim(S, P, ring, seq, (unsigned)kXmBlk * (unsigned)(P.pc_r * 128 + P.pc_r * 16));
            if (!dst) {
                ok = false;
                break;
            }
            unsigned long long *fb = &S.full[seq % (unsigned)ns];
            for (int bi = 0; bi < kXmBlk; ++bi) {
                const int b = q * kXmBlk + bi, rb = S.slot_e[j] * (P.H / 32) + (b >> 2);  // b: 8-row block
                tma_load_3d(dst + bi * P.dcb_r, mp + kMapDownQ, 32 * (b & 3), 0, rb, fb);
                tma_load_3d(dst + kXmBlk * P.dcb_r + bi * P.sbd_r, mp + kMapDownSb, 8 * (b & 3), 0, rb, fb);
            }
            ++seq;
        }
    }
    // let this thread's copies land before the CTA ends (bounded)
    for (unsigned q = seq > (unsigned)ns ? seq - (unsigned)ns : 0u; q < seq; ++q)
        mbar_drain(&S.full[q % (unsigned)ns], (q / (unsigned)ns) & 1u);
    if (a_issued > 0)
        for (int i = 0; i <= min(cw.nshg, P.ua); ++i) mbar_drain(&S.afull[i], (unsigned)(a_issued - 1) & 1u);
}

// ------------------------------------------------------------------ kernel

template <int NT, bool MMA>
__global__ void __launch_bounds__(kThreads, 1) decode_stack_kernel(const __grid_constant__ Params Pk) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Shared &S = *reinterpret_cast<Shared *>(base);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxSlots; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], 1);
        }
        for (int i = 0; i < kMaxA; ++i) mbar_init(&S.afull[i], 1);
        mbar_init(&S.aempty, 1u + (unsigned)min(cta_work(Pk.c).nshg, Pk.c.ua));  // router + static shared units
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i < (int)(sizeof(Cfg) / 4); i += blockDim.x)
        reinterpret_cast<unsigned *>(&S.c)[i] = reinterpret_cast<const unsigned *>(&Pk.c)[i];
    for (int i = threadIdx.x; i < kMaxA; i += blockDim.x) S.acnt[i] = 0;
    for (int i = threadIdx.x; i < kMaxSlots; i += blockDim.x) {
        S.owner[i] = 0xffffffffu;
        S.cnt[i] = 0;
        S.astate[i] = 0;
    }
    for (int i = threadIdx.x; i < 1 + kMaxPairs; i += blockDim.x) S.exp_ready[i] = 0u;
    for (int i = threadIdx.x; i < kMaxPairs; i += blockDim.x) S.pos_idx[i] = i;
    for (int i = threadIdx.x; i < kMaxT; i += blockDim.x) S.toks_sh[i] = i;
    if (threadIdx.x == 0) {
        S.tables_layer = 0;
        S.verdict = 1;
    }
    __syncthreads();
    if ((threadIdx.x >> 5) == kProdWarp) {
        producer_main<MMA>(Pk, S, base);  // lane 0 works, the other lanes return at once
        __syncwarp();
    } else {
        consumer_main<NT, MMA>(Pk, S, base);
    }
    __syncthreads();
}

}  // namespace dec

// ------------------------------------------------------------------ host side

namespace {

size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DecodeWs {
    size_t ctl, ready, zero_bytes, logits, a_sh, a_r, m, y_r, maps, total;
};

// Workspace: control words (barrier counters 128 bytes apart; the status word
// at byte 4), readiness counts, logits, SwiGLU outputs, m, tensor maps.
DecodeWs decode_ws(const moe_layer_w *w, int T) {
    DecodeWs d;
    size_t off = 0;
    auto take = [&](size_t b, size_t a = 256) {
        off = al(off, a);
        const size_t o = off;
        off += b;
        return o;
    };
    d.ctl = take(2048);
    d.ready = take(sizeof(unsigned) * (1 + dec::kMaxPairs));
    d.logits = take(2 * sizeof(unsigned long long) * (size_t)T * w->E);  // flag-in-data words: zeroed per launch
    d.zero_bytes = al(off, 256);
    d.a_sh = take(sizeof(float) * (size_t)T * w->Is);
    d.a_r = take(sizeof(float) * (size_t)T * w->k * w->I);
    d.m = take(sizeof(float) * (size_t)T * w->H);
    d.maps = take(sizeof(CUtensorMap) * dec::kMaxLayers * dec::kMaps, 128);
    // expert-major down (T >= 4 only): routed outputs by pair.  Below that the workspace keeps its size
    // (and its control words their placement: one 90 KB larger at T = 1 timed 1.5 % slower)
    d.y_r = take(T >= 4 ? sizeof(float) * (size_t)T * w->k * w->H : 0);
    d.total = al(off, 256);
    return d;
}

// K-parts of a down matrix with K input columns: parts of at most
// kPartChunks chunks, an even number of chunks each (whole groups).
void down_parts(int K, int *parts, int *pc) {
    const int C = K / 32, Gk = K / 64;
    int n = (C + dec::kPartChunks - 1) / dec::kPartChunks;
    *parts = n;
    *pc = 2 * ((Gk + n - 1) / n);
}

// The kernel's shared-memory plan for layers shaped like w, T tokens, a grid
// of `grid` CTAs; false if it does not fit.
bool decode_plan_xm(const moe_layer_w &w, int T, int grid, bool mma, bool allow_xm, dec::Cfg &P, size_t *smem) {
    if (grid <= 0 || T < 1 || T > dec::kMaxT || (long)T * w.H > dec::kMaxStageTH || w.H > 4096) return false;
    if ((long)T * w.k > dec::kMaxPairs) return false;
    P.H = w.H;
    P.E = w.E;
    P.k = w.k;
    P.I = w.I;
    P.Is = w.Is;
    P.T = T;
    P.CH = w.H / 32;
    P.GH = w.H / 64;
    P.units_s = w.Is / 8;
    P.units_r = w.I / 8;
    P.nrb8 = w.H / 8;
    down_parts(w.Is, &P.parts_s, &P.pc_s);
    down_parts(w.I, &P.parts_r, &P.pc_r);
    if (P.parts_s > dec::kMaxParts || P.parts_r > dec::kMaxParts) return false;
    const int nblk_max = (P.nrb8 + grid - 1) / grid;
    if (nblk_max > dec::kMaxBlk) return false;
    P.gcb = (int)al((size_t)P.CH * 128, 1024);
    P.sbs = (int)al((size_t)P.GH * 32, 128);
    P.dcb_s = (int)al((size_t)P.pc_s * 128, 1024);
    P.dcb_r = (int)al((size_t)P.pc_r * 128, 1024);
    P.sbd_s = (int)al((size_t)P.pc_s * 16, 128);
    P.sbd_r = (int)al((size_t)P.pc_r * 16, 128);
    const size_t g_slot = 2 * (size_t)P.gcb + 2 * (size_t)P.sbs;
    auto d_slot = [&](int dcb, int sbd, int pc) {
        const size_t area = mma ? (size_t)T * dec::ahl_token_bytes(pc) + (size_t)T * (pc / 2) * 4
                                : (size_t)T * pc * (dec::kXStride + 1) * 4;
        return (size_t)nblk_max * (dcb + sbd) + area;
    };
    const long nrows_r = (w.E + grid - 1) / grid;
    const size_t r_slot = 2 * (size_t)w.H + nrows_r * w.H + 2 * al(nrows_r * P.GH * 2 + 32, 16);
    // static region: the router rows and this CTA's shared gate/up units of one layer
    const int nshg_max = (P.units_s + grid - 1) / grid;
    P.a_rbytes = (int)al(r_slot, 1024);
    P.a_ubytes = (int)al(g_slot, 1024);
    // from 4 tokens on, the tensor-core variant does the routed down work by expert: a CTA takes a run
    // of (expert, 32-row block) items and stages each of its experts' input once; it needs one K-part per
    // routed down matrix, and room for the experts a run can reach (measured: T = 8 1592 -> 1948 tok/s,
    // T = 4 1630 -> 1716 on the Qwen-35B shape; T = 2 slower, 1270 -> 1203)
    P.xm = 0;
    P.ipe = w.H / (8 * dec::kXmBlk);
    P.nstage = 0;
    P.stage_bytes = 0;
    if (allow_xm && mma && T >= 4 && P.parts_r == 1 && w.H % (8 * dec::kXmBlk) == 0) {
        const long dmax = std::min((long)w.E, (long)T * w.k);
        const long itmax = (dmax * P.ipe + grid - 1) / grid;
        const long reach = (itmax + P.ipe - 1) / P.ipe + 1;
        if (reach <= dec::kMaxStage) {
            P.xm = 1;
            P.nstage = (int)reach;
            P.stage_bytes = (int)al((size_t)T * dec::ahl_token_bytes(P.pc_r) + (size_t)T * (P.pc_r / 2) * 4, 128);
        }
    }
    // ring: routed gate/up units and down groups (by output rows, or by expert)
    size_t slot = g_slot;
    slot = std::max(slot, d_slot(P.dcb_s, P.sbd_s, P.pc_s));
    if (P.xm)
        slot = std::max(slot, (size_t)dec::kXmBlk * (P.dcb_r + P.sbd_r));
    else
        slot = std::max(slot, d_slot(P.dcb_r, P.sbd_r, P.pc_r));
    P.slot_bytes = (int)al(slot, 1024);
    if ((w.E + 31) / 32 > dec::kMaxSl) return false;
    P.yrows = 8 * dec::kMaxBlk;
    // after the fixed part: static region and ring (1024-aligned), x, xs, h, ybuf, partials
    size_t off = al(sizeof(dec::Shared), 1024);
    P.off_a = (int)off;
    const size_t x_bytes = mma ? (size_t)T * dec::xb_token_bytes(P.CH) : (size_t)T * P.CH * dec::kXStride * 4;
    const size_t xs_bytes = mma ? (size_t)T * P.GH * 4 : (size_t)T * P.CH * 4;
    const size_t part_per_slot = mma ? (size_t)dec::kMaxPieces * 128 * 4 : (size_t)dec::kFfmaPart * 4;
    const size_t stage_all = (size_t)P.nstage * P.stage_bytes;
    // down outputs of this CTA's rows: routed by pair and shared, or (by expert) the shared ones only
    const size_t ybuf_bytes = (size_t)((P.xm ? 0 : T * w.k * P.parts_r) + P.parts_s * T) * P.yrows * 4;
    const size_t fixed_tail = al(x_bytes, 16) + al(xs_bytes, 16) + al((size_t)T * w.H * 2, 16) +
                              al(ybuf_bytes, 16) + (stage_all ? stage_all + 128 : 0);
    const size_t budget = 227 * 1024 - 1024;  // the base is aligned to 1024 bytes inside the allocation
    // as many of a CTA's shared units in the static region as leave the ring 3 slots or more; else none,
    // and 2 ring slots (every ring task is consumed in its own layer, so 2 slots cannot deadlock)
    size_t ring_min = 3 * ((size_t)P.slot_bytes + part_per_slot);
    int ua = std::min(nshg_max, dec::kMaxA - 1);
    auto a_need = [&](int u) { return (size_t)P.a_rbytes + (size_t)u * (P.a_ubytes + part_per_slot); };
    while (ua > 0 && off + a_need(ua) + fixed_tail + ring_min > budget) --ua;
    if (off + a_need(ua) + fixed_tail + ring_min > budget) ring_min = 2 * ((size_t)P.slot_bytes + part_per_slot);
    if (off + a_need(ua) + fixed_tail + ring_min > budget) return false;
    P.ua = ua;
    const size_t a_parts = (size_t)ua * part_per_slot;  // the static shared units' partial sums
    off += (size_t)P.a_rbytes + (size_t)ua * P.a_ubytes;
    P.off_ring = (int)off;
    long ns = (long)((budget - off - fixed_tail - a_parts) / ((size_t)P.slot_bytes + part_per_slot));
    if (ns > dec::kMaxSlots) ns = dec::kMaxSlots;
    P.ns = (int)ns;
    off += (size_t)ns * P.slot_bytes;
    P.off_x = (int)off;
    off += al(x_bytes, 16);
    P.off_xs = (int)off;
    off += al(xs_bytes, 16);
    P.off_h = (int)off;
    off += al((size_t)T * w.H * 2, 16);
    P.off_y = (int)off;
    off += al(ybuf_bytes, 16);
    P.off_part = (int)off;
    off += (size_t)ns * part_per_slot + a_parts;  // ring slots' partials, then the shared units'
    if (stage_all) off = al(off, 128);
    P.off_stage = (int)off;
    off += stage_all;
    *smem = off + 1024;
    return *smem <= 227 * 1024;
}

// The plan with the routed down work by expert where it fits, else by output rows.
bool decode_plan(const moe_layer_w &w, int T, int grid, bool mma, dec::Cfg &P, size_t *smem) {
    return decode_plan_xm(w, T, grid, mma, true, P, smem) || decode_plan_xm(w, T, grid, mma, false, P, smem);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A tiled matrix set as a 3-D tensor of 32-bit words: [n_rb][per_rb][words],
// boxes of {bx words, by, 1}.
cudaError_t make_map(CUtensorMap *m, const uint32_t *ptr, int words, int per_rb, int n_rb, int bx, int by,
                     bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)words, (cuuint64_t)per_rb, (cuuint64_t)n_rb};
    const cuuint64_t strides[2] = {(cuuint64_t)words * 4, (cuuint64_t)words * 4 * per_rb};
    const cuuint32_t box[3] = {(cuuint32_t)bx, (cuuint32_t)by, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The 12 tensor maps of one layer (see the kMap* enumeration).
cudaError_t layer_maps(const moe_layer_w &w, const dec::Cfg &P, CUtensorMap *m) {
    const int CH = w.H / 32, GH = w.H / 64, rr = w.E * w.I / 32, rs = w.Is / 32, rd = w.E * w.H / 32, rds = w.H / 32;
    cudaError_t e;
    if ((e = make_map(&m[dec::kMapGateQ], w.gate.q, 128, CH, rr, 32, CH, true)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapUpQ], w.up.q, 128, CH, rr, 32, CH, true)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapGateSb], w.gate.sb, 32, GH, rr, 8, GH, false)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapUpSb], w.up.sb, 32, GH, rr, 8, GH, false)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapShGateQ], w.sh_gate.q, 128, CH, rs, 32, CH, true)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapShUpQ], w.sh_up.q, 128, CH, rs, 32, CH, true)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapShGateSb], w.sh_gate.sb, 32, GH, rs, 8, GH, false)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapShUpSb], w.sh_up.sb, 32, GH, rs, 8, GH, false)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapDownQ], w.down.q, 128, w.I / 32, rd, 32, P.pc_r, true)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapDownSb], w.down.sb, 32, w.I / 64, rd, 8, P.pc_r / 2, false)) != cudaSuccess) return e;
    if ((e = make_map(&m[dec::kMapShDownQ], w.sh_down.q, 128, w.Is / 32, rds, 32, P.pc_s, true)) != cudaSuccess)
        return e;
    return make_map(&m[dec::kMapShDownSb], w.sh_down.sb, 32, w.Is / 64, rds, 8, P.pc_s / 2, false);
}

// Host copies of the tensor maps of recent layer sets (a stack's maps are
// encoded once and copied into the workspace on every launch).
struct MapCache {
    std::mutex mu;
    struct Entry {
        std::vector<moe_layer_w> key;
        int pc_s = 0, pc_r = 0;
        CUtensorMap *host = nullptr;  // pinned, L * kMaps maps
        cudaEvent_t copied = nullptr;  // after the last copy out of `host`
        unsigned long long used = 0;
    };
    Entry entries[8];
    unsigned long long tick = 0;
};
MapCache g_maps;

bool same_layers(const std::vector<moe_layer_w> &a, const moe_layer_w *b, int L) {
    return (int)a.size() == L && std::memcmp(a.data(), b, sizeof(moe_layer_w) * L) == 0;
}

// Copies the maps of `layers` into the workspace (`dst`) on stream st,
// encoding them first unless a recent launch used the same layer set.
cudaError_t copy_maps(const moe_layer_w *layers, int L, const dec::Cfg &P, void *dst, cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g_maps.mu);
    MapCache::Entry *hit = nullptr, *victim = &g_maps.entries[0];
    for (auto &en : g_maps.entries) {
        if (en.host && en.pc_s == P.pc_s && en.pc_r == P.pc_r && same_layers(en.key, layers, L)) hit = &en;
        if (en.used < victim->used) victim = &en;
    }
    if (!hit) {
        hit = victim;
        if (!hit->host) {
            cudaError_t e = cudaMallocHost(&hit->host, sizeof(CUtensorMap) * dec::kMaxLayers * dec::kMaps);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hit->copied, cudaEventDisableTiming);
            if (e != cudaSuccess) {
                if (hit->host) cudaFreeHost(hit->host);
                hit->host = nullptr;
                return e;
            }
        } else {
            // an earlier launch may still be copying out of this entry
            cudaError_t e = cudaEventSynchronize(hit->copied);
            if (e != cudaSuccess) return e;
        }
        hit->key.assign(layers, layers + L);
        hit->pc_s = P.pc_s;
        hit->pc_r = P.pc_r;
        for (int l = 0; l < L; ++l) {
            cudaError_t e = layer_maps(layers[l], P, hit->host + (size_t)l * dec::kMaps);
            if (e != cudaSuccess) {
                hit->key.clear();
                return e;
            }
        }
    }
    hit->used = ++g_maps.tick;
    cudaError_t e = cudaMemcpyAsync(dst, hit->host, sizeof(CUtensorMap) * dec::kMaps * L, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaEventRecord(hit->copied, st);
    return e;
}

template <int NT, bool MMA>
const void *kernel_ptr() {
    return reinterpret_cast<const void *>(dec::decode_stack_kernel<NT, MMA>);
}

// The tensor-core variants for T >= 2 (the CUDA cores' FMA work grows with T,
// the MMA's does not), the CUDA-core FMAs for one token; force_path overrides.
bool use_mma(int T, int force_path) { return force_path >= 2 || (force_path == 0 && T >= 2); }

const void *kernel_for(int T, bool mma) {
    if (mma) return kernel_ptr<8, true>();
    if (T <= 1) return kernel_ptr<1, false>();
    if (T <= 2) return kernel_ptr<2, false>();
    if (T <= 4) return kernel_ptr<4, false>();
    return kernel_ptr<8, false>();
}

}  // namespace

size_t decode_stack_ws_bytes(const moe_layer_w *w, int T) { return decode_ws(w, T).total; }

size_t decode_stack_status_offset() { return sizeof(unsigned); }

bool decode_stack_fits(const moe_layer_w *w, int T, int grid, int force_path) {
    dec::Cfg P{};
    size_t smem = 0;
    return decode_plan(*w, T, grid, use_mma(T, force_path), P, &smem);
}

int decode_stack_max_tokens() { return dec::kMaxT; }
int decode_stack_max_layers() { return dec::kMaxLayers; }
int decode_stack_stage_floats() { return dec::kMaxStageTH; }

cudaError_t launch_decode_stack(const moe_layer_w *layers, int L, const uint16_t *h_in, int chained,
                                uint16_t *h_out, int T, void *ws, const moe_opts &o, int grid, cudaStream_t st) {
    const moe_layer_w &w = layers[0];
    const DecodeWs d = decode_ws(&w, T);
    dec::Params Pk;  // ~10 KiB, passed by value (kernel parameters up to 32 KiB)
    dec::Cfg &P = Pk.c;
    std::memset(&P, 0, sizeof P);
    size_t smem = 0;
    const bool mma = use_mma(T, o.force_path);
    if (!decode_plan(w, T, grid, mma, P, &smem)) return cudaErrorInvalidValue;
    for (int l = 0; l < L; ++l) Pk.layers[l] = layers[l];
    P.h_in = h_in;
    P.h_out = h_out;
    P.L = L;
    P.chained = chained;
    P.post_norm = o.post_norm;
    P.layer_scalar = o.layer_scalar;
    P.eps = o.eps;
    char *base = static_cast<char *>(ws);
    P.bar = reinterpret_cast<unsigned *>(base + d.ctl);
    // test hook: MOE_TEST_BARRIER_EXTRA=1 makes the grid barriers wait for one
    // arrival more than the grid has, so that the first one's bounded wait runs
    // out (about 1 s) and the kernel reports "grid barrier timed out" through
    // the workspace status
    const char *extra = getenv("MOE_TEST_BARRIER_EXTRA");
    P.bar_extra = (extra && extra[0] == '1') ? 1u : 0u;
    P.err = reinterpret_cast<int *>(base + d.ctl + sizeof(unsigned));
    P.ready = reinterpret_cast<unsigned *>(base + d.ready);
    P.logit_ll = reinterpret_cast<unsigned long long *>(base + d.logits);
    P.a_sh = reinterpret_cast<float *>(base + d.a_sh);
    P.a_r = reinterpret_cast<float *>(base + d.a_r);
    P.m = reinterpret_cast<float *>(base + d.m);
    P.y_r = reinterpret_cast<float *>(base + d.y_r);
    P.maps = reinterpret_cast<const CUtensorMap *>(base + d.maps);

    const void *fn = kernel_for(T, mma);
    cudaError_t e = ensure_smem(fn, smem);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(ws, 0, d.zero_bytes, st)) != cudaSuccess) return e;
    if ((e = copy_maps(layers, L, P, base + d.maps, st)) != cudaSuccess) return e;
    void *args[] = {&Pk};
    return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(dec::kThreads), args, smem, st);
}

cudaError_t decode_stack_grid(int device, int *grid) {
    int sms = 0, per = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) return e;
    // the largest plan any launch may use: one CTA per SM must fit
    const size_t smem = 227 * 1024;
    const void *fns[5] = {kernel_ptr<1, false>(), kernel_ptr<2, false>(), kernel_ptr<4, false>(), kernel_ptr<8, false>(),
                          kernel_ptr<8, true>()};
    for (const void *fn : fns) {
        if ((e = ensure_smem(fn, smem)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, dec::kThreads, smem)) != cudaSuccess) return e;
        if (per < 1) {
            *grid = 0;
            return cudaSuccess;
        }
    }
    *grid = sms;
    return cudaSuccess;
}

size_t decode_stack_smem() { return 227 * 1024; }

}  // namespace moe
