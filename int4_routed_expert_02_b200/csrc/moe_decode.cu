// moe_decode.cu -- persistent decode kernel: a stack of MoE layers for a small
// token batch (T <= 8) in ONE cooperative launch, one CTA per SM.
//
// Per layer (TurboFieldfare introduction page, discuss.pytorch.kr, section
// "TurboFieldfare's expert streaming structure": router -> routed experts +
// shared expert -> weighted combine -> normalisation, residual, layer scalar;
// weights MLX affine, section "How TurboFieldfare saves memory"):
//
//   P0  finish the previous layer: m = sum_s w_s y_s + shared, post-norm,
//       residual, layer scalar (every CTA, redundantly; CTA 0 writes it out),
//       and the RMS the router needs
//   P1  router logits in fp64 for this CTA's share of the E experts; its
//       router rows and router_scale were bulk-copied into shared memory at
//       the start of the layer, overlapping P0
//   --- grid barrier ---
//   P2  top-k + softmax * per_expert_scale and bucketing, by rank counting
//       (every CTA, redundantly, so no barrier is needed before the experts),
//       and this CTA's job tables for the two expert phases
//   P2' gate/up: a job (32 rows: a row block of one slot) is split into
//       tasks of <= 16 quantisation groups of one matrix; tasks are dealt
//       round-robin to the CTAs and taken by teams of kWPT warps (every
//       kWPT-th group each) independently; each warp's partial sums go to
//       global memory, and the warp that
//       finishes a job's last share (an atomic count per job) sums the parts
//       in a fixed order and forms a = silu(g) * u for the job's rows, then
//       counts the job done for its slot
//   (no grid barrier: a CTA stages a slot's input once all of that slot's
//   jobs are counted)
//   P3  down: tasks of 32 rows x <= 16 groups of one slot, in contiguous
//       blocks per CTA so that a CTA stages each slot's a once; each warp of
//       a task's team writes its partial rows, and the warp that finishes the
//       last share of a row block (an atomic count per row block) forms the combine
//       m = sum_s w_s y_s + shared for those rows, then counts the row block
//       done
//   (no grid barrier: the next layer's P0 waits until every row block of m
//   is counted)
//
// Weights stream HBM -> shared memory with 1-D bulk copies (cp.async.bulk)
// into a ring of mbarrier-guarded slots, one slot per task, issued by one
// producer thread ahead of 15 consumer warps (teams of kWPT = 1) that never
// wait for one another inside a phase.  The down tasks' weights do not depend on the gate/up
// results, so the producer already fills the slots freed during the gate/up
// phase with them.  Once the top-k is known each CTA also asks L2 to
// prefetch the down-projection weights of its later jobs, and during the down
// phase its share of the next layer's shared-expert weights, so HBM keeps
// streaming across the grid barriers.  The dot products use the subnormal
// code decode of moe_common.cuh (one AND + one FMA per code).  Loops keep the
// special-function pipe idle: no runtime integer division, conversion or
// reciprocal per element (job tables are built once per layer, the ring
// position is advanced incrementally, bf16 rounding uses integer arithmetic).
//
// Every wait is bounded (grid barrier and mbarriers: ~1 s of globaltimer); on
// a timeout the kernel records an error code in the workspace, stops taking
// work, lets its own bulk copies land and returns.
#include <cstdlib>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace dec {

constexpr int kCWarps = 15;                   // consumer warps: with the producer 16 warps, 4 per SM sub-partition,
                                              // so a thread may hold 128 registers (no spills)
constexpr int kWPT = 1;                       // consumer warps per task (a team; more than one measured slower)
constexpr int kTeams = kCWarps / kWPT;
constexpr int kWarps = kCWarps + 1;           // + the producer warp
constexpr int kThreads = kWarps * 32;
constexpr int kProducerWarp = kCWarps;
constexpr int kMaxStages = 11;                // ring slots: as many as fit beside the input stage
constexpr int kTaskGroups = 16;               // groups per task (one ring slot)
constexpr int kCodeBytesPerGroup = 1024;      // 32 rows x 64 codes x 4 bits
constexpr int kSbBytesPerGroup = 128;         // 32 rows x (scale, bias)
constexpr int kSlotBytes = 16 * (kCodeBytesPerGroup + kSbBytesPerGroup);  // 18432
constexpr int kMaxT = 8;
constexpr int kStageFloats = 24576;           // largest input stage (T * H)
constexpr int kPoolBytes = 11 * kSlotBytes;   // ring + input stage share this pool
constexpr int kMaxXs = 768;
constexpr int kMaxLayers = 64;
constexpr int kMaxPairs = kMaxT * kMaxK;
constexpr int kMaxTasks = 160;                // per CTA and phase
constexpr int kMaxPG = 4;                     // gate/up parts per job (H <= 4096)
constexpr int kMaxSegs = 16;                  // down: staged (slot, part) inputs per CTA
constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s

constexpr int kErrGridBarrier = 1, kErrFull = 2, kErrEmpty = 3, kErrReady = 4;

// Sizes, options and workspace pointers of a launch.  The kernel copies them
// into shared memory once, so that every phase reads them at shared-memory
// latency instead of through the kernel-parameter space.
struct Cfg {
    const uint16_t *h_in;  // [T,H] (chained) or [L,T,H]
    uint16_t *h_out;       // [L,T,H]: every layer's output
    int L, T, chained, post_norm;
    float layer_scalar, eps;
    int H, E, k, I, Is, Kmax, R;
    int ndp_r, ndp_s;
    int nslots;      // ring slots (the rest of the pool is the input stage)
    int stage_floats;  // floats in the input stage
    unsigned *bar;
    unsigned bar_extra;  // arrivals the grid barrier waits for beyond the grid (0; tests of the timeout path set 1)
    int *err;
    unsigned *cnt_dn;  // [H/32]: down tasks done per row block; reset by the last
    unsigned *cnt_gu;  // [jobs]: gate/up tasks done per job; reset by the last
    unsigned *act_done;   // [1 + T*k]: gate/up jobs done per slot, over all layers so far
    unsigned *rows_done;  // row blocks of m combined, over all layers so far
    float *gpart;      // [jobs][2][pg][kWPT][T][32]: gate/up partial sums per task member
    double *logits;  // [T,E]
    float *act;      // [R][Kmax]: SwiGLU output a per rowset (shared tokens, then bucketed pairs),
                     // pre-scaled for the code decode
    float *act_cs;   // [R][Kmax/32]: sums of a over 32-column chunks
    float *y;        // [ndp_r * kWPT][T*k][H]: down partial sums per task member
    float *sh;       // [ndp_s * kWPT][T][H]
    float *m;        // [T][H]: the combine m of the current layer
};

struct Params {
    Cfg c;
    moe_layer_w layers[kMaxLayers];
};

// One task of an expert phase: 32 rows (row block rb) x groups [g0, g1) of
// matrix mat (gate/up: 0 gate, 1 up; down: 0) of the shared expert (slot 0)
// or of routed expert e (slot >= 1), for n tokens starting at bucketed
// position seg0.  job: gate/up, the CTA-local job; seg: down, the staged input.
struct TaskDesc {
    int16_t slot, rb, mat, part, g0, g1, n, seg;
    int32_t seg0, e, job;
};

// A staged down-phase input: the SwiGLU rows of one (slot, part), columns
// [g0*64, g0*64 + ld), token tt at stage offset off + tt * ld.
struct SegDesc {
    int16_t slot, part, n, g0, ld, pad;
    int32_t seg0, off;
};

struct Smem {
    alignas(128) unsigned char pool[kPoolBytes];  // ring slots, then the input stage
    alignas(8) unsigned long long full[kMaxStages];
    alignas(8) unsigned long long empty[kMaxStages];
    alignas(8) unsigned long long rbar;  // router copies of the current layer
    unsigned slot_task[kMaxStages];      // ring sequence number of the task a slot currently holds
    float *stage;                        // input stage (inside the pool, after the ring)
    alignas(16) float xs[kMaxXs];        // sum of x per 32-column chunk
    float bred[32];  // block reductions
    TaskDesc gut[kMaxTasks], dnt[kMaxTasks];
    SegDesc seg[kMaxSegs];
    int ngt, ndt, pg, nseg, seg_rounds;
    unsigned act_expect[kMaxPairs + 1];  // act_done per slot once this layer's gate/up jobs are all done
    double selv[kMaxPairs];
    float wts[kMaxPairs];
    int idx[kMaxPairs];
    int perm[kMaxPairs];
    int act_e[kMaxPairs], act_off[kMaxPairs], act_n[kMaxPairs];
    int poff[kMaxPairs], pcnt[kMaxPairs];
    unsigned char first[kMaxPairs];
    int tokrow[kMaxPairs];  // bucketed position j -> row offset (token * H) of its input
    int tokrow_sh[kMaxT];   // shared expert: token t -> t * H
    int nact;
    double rpart[128];
    float rms[kMaxT];
    float rinv[kMaxT];
    int rcopy[3];  // router copies of this layer: first row, rows, byte offset of the scale/bias superset
    int flag;
    int flag2;  // consumer-only verdicts
    Cfg c;          // the launch's Cfg
    moe_layer_w w;  // the current layer's weights
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Block-cooperative copy of a 4-byte-aligned struct (no barrier).
__device__ __forceinline__ void copy_words(void *dst, const void *src, size_t bytes) {
    for (int i = threadIdx.x; i < (int)(bytes / 4); i += blockDim.x)
        static_cast<unsigned *>(dst)[i] = static_cast<const unsigned *>(src)[i];
}

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

// Bounded wait for the phase with `parity` of mbarrier `b` to complete.
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

// Bounded wait used only when draining: ignores the error flag.
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

// Prefetch [p, p + bytes) into L2 in pieces of at most 64 KiB (16-byte units).
__device__ __forceinline__ void prefetch_range(const void *p, size_t bytes) {
    const char *c = static_cast<const char *>(p);
    while (bytes >= 16) {
        const unsigned n = (unsigned)(bytes > 65536 ? 65536 : (bytes & ~(size_t)15));
        prefetch_l2(c, n);
        c += n;
        bytes -= n;
    }
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCWarps * 32) : "memory"); }

// Grid-wide barrier number `nth` (1, 2, ...) on a monotonically increasing
// counter; bounded.  Returns false (in every thread of the CTA alike) if any
// CTA recorded an error.
__device__ __noinline__ bool grid_sync(const Cfg &P, unsigned nth, int *verdict) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(P.bar, 1u);
        const unsigned target = nth * gridDim.x + P.bar_extra;
        const unsigned long long t0 = globaltimer();
        for (unsigned it = 0;; ++it) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(P.bar) : "memory");
            if (v >= target) break;
            if ((it & 63u) == 63u) {
                if (ldcg_int(P.err) != 0) break;
                if (globaltimer() - t0 > kWaitNs) {
                    atomicCAS(P.err, 0, kErrGridBarrier);
                    break;
                }
            }
            __nanosleep(32);
        }
        __threadfence();
        *verdict = ldcg_int(P.err) == 0;
    }
    __syncthreads();
    return *verdict != 0;
}

// ------------------------------------------------------------------ jobs

// Task gt (grid-wide index; this CTA takes gt = c, c + G, ...) of the gate/up
// phase.  Job j = gt / (2 pg) is 32 rows of the shared expert or of one
// active slot; its 2 pg tasks are part p of gate and of up, p = 0..pg-1.
// All divisions happen here, once per task.
__device__ __forceinline__ TaskDesc make_gu_task(const Cfg &P, const Smem &S, int gt, int pg) {
    TaskDesc t;
    const int j = gt / (2 * pg), r = gt - j * 2 * pg;
    const int A = P.Is / 32;
    if (j < A) {
        t.slot = 0;
        t.rb = (int16_t)j;
        t.n = (int16_t)P.T;
        t.seg0 = 0;
        t.e = -1;
    } else {
        const int B = P.I / 32, jj = j - A, a = jj / B;
        t.slot = (int16_t)(1 + a);
        t.rb = (int16_t)(jj - a * B);
        t.seg0 = S.act_off[a];
        t.n = (int16_t)S.act_n[a];
        t.e = S.act_e[a];
    }
    const int GH = P.H / 64;
    t.mat = (int16_t)(r & 1);
    t.part = (int16_t)(r >> 1);
    t.g0 = (int16_t)(GH * t.part / pg);
    t.g1 = (int16_t)(GH * (t.part + 1) / pg);
    t.job = j;
    t.seg = 0;
    return t;
}

// (slot, part) number sp of the down phase: the shared expert's parts first,
// then each active slot's.
__device__ __forceinline__ void dn_slot_part(const Cfg &P, int sp, int &slot, int &part) {
    if (sp < P.ndp_s) {
        slot = 0;
        part = sp;
    } else {
        const int a = (sp - P.ndp_s) / P.ndp_r;
        slot = 1 + a;
        part = sp - P.ndp_s - a * P.ndp_r;
    }
}

// Task d (grid-wide index) of the down phase: (slot, part) d / (H/32), row block d % (H/32).
__device__ __forceinline__ TaskDesc make_dn_task(const Cfg &P, const Smem &S, int d, int sp0) {
    TaskDesc t;
    const int RBH = P.H / 32, sp = d / RBH;
    int slot, part;
    dn_slot_part(P, sp, slot, part);
    t.slot = (int16_t)slot;
    t.part = (int16_t)part;
    t.rb = (int16_t)(d - sp * RBH);
    t.mat = 0;
    const int G = slot == 0 ? P.Is / 64 : P.I / 64, nd = slot == 0 ? P.ndp_s : P.ndp_r;
    t.g0 = (int16_t)(G * part / nd);
    t.g1 = (int16_t)(G * (part + 1) / nd);
    if (slot == 0) {
        t.n = (int16_t)P.T;
        t.seg0 = 0;
        t.e = -1;
    } else {
        t.seg0 = S.act_off[slot - 1];
        t.n = (int16_t)S.act_n[slot - 1];
        t.e = S.act_e[slot - 1];
    }
    t.job = 0;
    t.seg = (int16_t)(sp - sp0);
    return t;
}

// Weight pointers (codes, scale/bias words) of a task's row block.
__device__ __forceinline__ void task_ptrs(const Cfg &P, const moe_layer_w &W, const TaskDesc &t, bool down,
                                          const uint32_t *&q, const uint32_t *&sb) {
    if (!down) {
        const size_t CH = P.H / 32, GH = P.H / 64;
        const moe_qmat &M = t.slot == 0 ? (t.mat ? W.sh_up : W.sh_gate) : (t.mat ? W.up : W.gate);
        const size_t mrb = t.slot == 0 ? (size_t)t.rb : (size_t)t.e * (P.I / 32) + t.rb;
        q = M.q + mrb * CH * 128;
        sb = M.sb + mrb * GH * 32;
    } else if (t.slot == 0) {
        q = W.sh_down.q + (size_t)t.rb * (P.Is / 32) * 128;
        sb = W.sh_down.sb + (size_t)t.rb * (P.Is / 64) * 32;
    } else {
        const size_t mrb = (size_t)t.e * (P.H / 32) + t.rb;
        q = W.down.q + mrb * (P.I / 32) * 128;
        sb = W.down.sb + mrb * (P.I / 64) * 32;
    }
}

// rowset of the tt-th token of a task (shared: the token; routed: T + bucketed position)
__device__ __forceinline__ int task_rowset(const Cfg &P, const TaskDesc &t, int tt) {
    return t.slot == 0 ? tt : P.T + t.seg0 + tt;
}

// Producer: the copies that fill ring slot s with groups [g0, g1) of one
// matrix: codes (ng KiB), then the (scale, bias) words (ng * 128 B).
__device__ __forceinline__ void issue_task(Smem &S, int s, const uint32_t *q, const uint32_t *sb, int g0, int g1) {
    const int ng = g1 - g0;
    const unsigned cb = (unsigned)ng * kCodeBytesPerGroup, sbb = (unsigned)ng * kSbBytesPerGroup;
    unsigned char *slot = S.pool + (size_t)s * kSlotBytes;
    mbar_expect_tx(&S.full[s], cb + sbb);
    bulk_g2s(slot, q + (size_t)g0 * 256, cb, &S.full[s]);
    bulk_g2s(slot + cb, sb + (size_t)g0 * 32, sbb, &S.full[s]);
}

// ------------------------------------------------------------------ dot products

// One (matrix, group) of a job for tokens [t0, t0 + n), n <= NT <= 2: lanes
// are the 32 rows.  w: this lane's 64 codes of the group; s (already times
// 2^49) and b: its scale and bias.  The input of token tt starts at
// x + off(tt), its chunk sums at xsum + off(tt) / 32, where off(tt) =
// tokrow[tt] (gathered tokens) or tt * stride (when tokrow is null).
template <int NT>
__device__ __forceinline__ void group_dot(const uint32_t (&w)[8], float s, float b, const float *x,
                                          const float *xsum, const int *tokrow, int stride, int t0, int n,
                                          float (&acc)[4]) {
    constexpr int NA = NT == 1 ? 2 : 1;  // packed accumulators per token: 2 for ILP when alone
    float2 a[NT][NA];
    int xo[NT];
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
#pragma unroll
        for (int z = 0; z < NA; ++z) a[tt][z] = make_float2(0.f, 0.f);
        xo[tt] = tt < n ? (tokrow ? tokrow[t0 + tt] : (t0 + tt) * stride) : 0;
    }
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
        const Decoded8 f = decode_word(w[wi]);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
            if (tt < n) {
                const float4 *x4 = reinterpret_cast<const float4 *>(x + xo[tt] + wi * 8);
                const float4 xa = x4[0], xb = x4[1];
                a[tt][0] = ffma2(make_float2(f.f[0], f.f[1]), make_float2(xa.x, xa.y), a[tt][0]);
                a[tt][NA - 1] = ffma2(make_float2(f.f[2], f.f[3]), make_float2(xa.z, xa.w), a[tt][NA - 1]);
                a[tt][0] = ffma2(make_float2(f.f[4], f.f[5]), make_float2(xb.x, xb.y), a[tt][0]);
                a[tt][NA - 1] = ffma2(make_float2(f.f[6], f.f[7]), make_float2(xb.z, xb.w), a[tt][NA - 1]);
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
        if (tt < n) {
            float d = a[tt][0].x + a[tt][0].y;
            if (NA == 2) d += a[tt][NA - 1].x + a[tt][NA - 1].y;
            const int c = xo[tt] >> 5;
            acc[tt] = fmaf(s, d, fmaf(b, xsum[c] + xsum[c + 1], acc[tt]));
        }
    }
}

// One (matrix, group) for the n <= NT tokens of a job, in calls of at most two
// tokens (codes are decoded once per call); acc[tt] is token tt's sum.
template <int NT>
__device__ __forceinline__ void group_dot_n(const unsigned char *codes, uint32_t sbw, const float *x,
                                            const float *xsum, const int *tokrow, int stride, int n,
                                            float (&acc)[NT], int lane) {
    const uint4 c0 = reinterpret_cast<const uint4 *>(codes)[lane];
    const uint4 c1 = reinterpret_cast<const uint4 *>(codes + 512)[lane];
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float s = bf16_bits_to_float(sbw & 0xffffu) * kCodeUnscale, b = bf16_bits_to_float(sbw >> 16);
    if (NT == 1) {
        float a4[4] = {acc[0], 0.f, 0.f, 0.f};
        group_dot<1>(w, s, b, x, xsum, tokrow, stride, 0, 1, a4);
        acc[0] = a4[0];
        return;
    }
#pragma unroll
    for (int t0 = 0; t0 < NT; t0 += 2) {
        if (t0 < n) {
            float p[4] = {acc[t0], t0 + 1 < NT ? acc[t0 + 1 < NT ? t0 + 1 : 0] : 0.f, 0.f, 0.f};
            group_dot<2>(w, s, b, x, xsum, tokrow, stride, t0, min(2, n - t0), p);
            acc[t0] = p[0];
            if (t0 + 1 < NT) acc[t0 + 1 < NT ? t0 + 1 : 0] = p[1];
        }
    }
}

// ------------------------------------------------------------------ phases

// Input rows of a layer straight from global memory (bf16) into S.stage, and their RMS.
__device__ __noinline__ void load_input(const Cfg &P, Smem &S, const uint16_t *h) {
    const int T = P.T, H = P.H, H2 = H / 2;
    float *stage = S.stage;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float ss = 0.f;
#pragma unroll 1
        for (int i = threadIdx.x; i < H2; i += blockDim.x) {
            const uint32_t v = __ldcg(reinterpret_cast<const unsigned int *>(h + (size_t)t * H) + i);
            const float a = bf16_bits_to_float(v & 0xffffu), b = bf16_bits_to_float(v >> 16);
            stage[(size_t)t * H + 2 * i] = a;
            stage[(size_t)t * H + 2 * i + 1] = b;
            ss = fmaf(a, a, fmaf(b, b, ss));
        }
        ss = block_sum(ss, S.bred);
        if (threadIdx.x == 0) {
            S.rms[t] = sqrtf(ss / (float)H + P.eps);
            S.rinv[t] = 1.0f / S.rms[t];
        }
    }
    __syncthreads();
}

// P0: output of layer lp (its combine m, post-norm, residual, scalar) into
// S.stage as floats, with its RMS; CTA 0 also writes it to h_out[lp].
// H/4 <= 1024 < 2 * blockDim, so two float4 per thread cover a row.
__device__ __noinline__ void finish_layer(const Cfg &P, Smem &S, int lp) {
    const int T = P.T, H = P.H, H4 = H / 4;
    const uint16_t *hprev = (P.chained && lp > 0) ? P.h_out + (size_t)(lp - 1) * T * H
                                                  : (P.chained ? P.h_in : P.h_in + (size_t)lp * T * H);
    uint16_t *out = P.h_out + (size_t)lp * T * H;
    float *stage = S.stage;
    const float scalar = P.layer_scalar;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float4 mreg[2];
        uint2 hreg[2];
        float ss = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i4 = threadIdx.x + r * blockDim.x;
            mreg[r] = make_float4(0.f, 0.f, 0.f, 0.f);
            hreg[r] = make_uint2(0u, 0u);
            if (i4 < H4) {
                hreg[r] = __ldcg(reinterpret_cast<const uint2 *>(hprev + (size_t)t * H) + i4);
                mreg[r] = __ldcg(reinterpret_cast<const float4 *>(P.m + (size_t)t * H) + i4);
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r)
            ss += mreg[r].x * mreg[r].x + mreg[r].y * mreg[r].y + mreg[r].z * mreg[r].z + mreg[r].w * mreg[r].w;
        ss = block_sum(ss, S.bred);
        const float inv = P.post_norm ? 1.0f / sqrtf(ss / (float)H + P.eps) : 1.0f;
        float ss2 = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i4 = threadIdx.x + r * blockDim.x;
            if (i4 < H4) {
                const float mv[4] = {mreg[r].x, mreg[r].y, mreg[r].z, mreg[r].w};
                const uint32_t hv[2] = {hreg[r].x, hreg[r].y};
                uint32_t o[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float hp = bf16_bits_to_float((hv[c >> 1] >> (16 * (c & 1))) & 0xffffu);
                    o[c] = f32_to_bf16_bits_alu((hp + mv[c] * inv) * scalar);
                    const float of = bf16_bits_to_float(o[c]);
                    stage[(size_t)t * H + 4 * i4 + c] = of;
                    ss2 = fmaf(of, of, ss2);
                }
                if (blockIdx.x == 0)
                    reinterpret_cast<uint2 *>(out + (size_t)t * H)[i4] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
            }
        }
        ss2 = block_sum(ss2, S.bred);
        if (threadIdx.x == 0) {
            S.rms[t] = sqrtf(ss2 / (float)H + P.eps);
            S.rinv[t] = 1.0f / S.rms[t];
        }
    }
    __syncthreads();
}

// Producer, at the start of layer l: router_scale, this CTA's router rows
// [e0, e1) and a 16-byte-aligned superset of their scales and biases, into
// the ring (idle until the top-k), completing on S.rbar (one phase per layer).
__device__ __noinline__ void issue_router_copies(const Cfg &P, Smem &S, const moe_layer_w &W) {
    const int E = P.E, H = P.H, G = H / 64;
    const int e0 = (int)((long long)E * blockIdx.x / gridDim.x), e1 = (int)((long long)E * (blockIdx.x + 1) / gridDim.x);
    const int nrows = e1 - e0;
    unsigned char *base = S.pool;
    const unsigned rs_bytes = (unsigned)H * 2, rows_bytes = (unsigned)nrows * H;
    const unsigned sb_lo = (unsigned)((size_t)e0 * G * 2) & ~15u;
    const unsigned sb_hi = ((unsigned)((size_t)e1 * G * 2) + 15u) & ~15u;
    const unsigned sb_bytes = nrows > 0 ? sb_hi - sb_lo : 0u;
    S.rcopy[0] = e0;
    S.rcopy[1] = nrows;
    S.rcopy[2] = (int)sb_lo;
    mbar_expect_tx(&S.rbar, rs_bytes + rows_bytes + 2 * sb_bytes);
    // layout: [router_scale (H*2)] [rows (nrows*H)] [scales (sb_bytes)] [biases (sb_bytes)]
    bulk_g2s(base, W.router_scale, rs_bytes, &S.rbar);
    if (nrows > 0) {
        bulk_g2s(base + rs_bytes, W.router_q + (size_t)e0 * (H / 4), rows_bytes, &S.rbar);
        bulk_g2s(base + rs_bytes + rows_bytes, reinterpret_cast<const char *>(W.router_s) + sb_lo, sb_bytes, &S.rbar);
        bulk_g2s(base + rs_bytes + rows_bytes + sb_bytes, reinterpret_cast<const char *>(W.router_b) + sb_lo, sb_bytes,
                 &S.rbar);
    }
}

// P1: router logits of this CTA's experts for every token, from the copies in
// the ring.  The dot products accumulate in fp64 so that the top-k order does
// not depend on summation order; the common factor 1 / (rms * sqrt(H)) of a
// token's logits is applied last (it cannot change their order).
__device__ __noinline__ void router_phase(const Cfg &P, Smem &S, int l) {
    const int T = P.T, H = P.H, E = P.E, G = H / 64, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    __syncthreads();  // S.rcopy written by the producer thread
    const int e0 = S.rcopy[0], nrows = S.rcopy[1], sb_lo = S.rcopy[2];
    const int items = nrows * T;
    // every thread waits for the copies (they are issued even when nrows == 0);
    // the verdict is made uniform before the barriers below
    const bool got = __syncthreads_and(mbar_wait(&S.rbar, (unsigned)(l & 1), P.err, kErrFull)) != 0;
    const unsigned char *base = S.pool;
    const uint16_t *rsc = reinterpret_cast<const uint16_t *>(base);
    const unsigned rows_bytes = (unsigned)nrows * H;
    const unsigned sb_hi = ((unsigned)((size_t)(e0 + nrows) * G * 2) + 15u) & ~15u;
    const unsigned sb_bytes = nrows > 0 ? sb_hi - (unsigned)sb_lo : 0u;
    const unsigned char *rows = base + H * 2;
    const int sb_skip = (int)((size_t)e0 * G * 2) - sb_lo;
    const uint16_t *scs = reinterpret_cast<const uint16_t *>(rows + rows_bytes + sb_skip);
    const uint16_t *bis = reinterpret_cast<const uint16_t *>(rows + rows_bytes + sb_bytes + sb_skip);
    if (items > 0 && got) {
        const int parts = items >= kWarps ? 1 : kWarps / items;
        const int units = items * parts;
        const int nch = H / 16;
        const float *stage = S.stage;
#pragma unroll 1
        for (int u = wid; u < units; u += kWarps) {
            const int item = u / parts, part = u - item * parts;
            const int er = item / T, t = item - er * T;
            const int c0 = nch * part / parts, c1 = nch * (part + 1) / parts;
            const float *h = stage + (size_t)t * H;
            double acc = 0.0;
#pragma unroll 1
            for (int c = c0 + lane; c < c1; c += 32) {
                const uint4 q = reinterpret_cast<const uint4 *>(rows + (size_t)er * H)[c];
                const uint32_t words[4] = {q.x, q.y, q.z, q.w};
                double dots[4] = {0.0, 0.0, 0.0, 0.0}, zss[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                    for (int bi = 0; bi < 4; ++bi) {
                        const int i = c * 16 + wi * 4 + bi;
                        // h * router_scale is exact in fp32 (two bf16 values)
                        const double z = (double)(h[i] * bf16_bits_to_float(rsc[i]));
                        // the 8-bit code as a double: 2^52 + q read as fp64, minus 2^52 (exact)
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
            if (lane == 0) S.rpart[u] = acc;
        }
        __syncthreads();
        const double sqrt_h = sqrt((double)H);
#pragma unroll 1
        for (int item = threadIdx.x; item < items; item += blockDim.x) {
            double a = 0.0;
            for (int p = 0; p < parts; ++p) a += S.rpart[item * parts + p];
            const int er = item / T, t = item - er * T;
            P.logits[(size_t)t * E + e0 + er] = a / ((double)S.rms[t] * sqrt_h);
        }
    }
    __syncthreads();
}

// P2: top-k by rank counting (a logit's rank = how many logits beat it: larger,
// or equal with a lower expert index), softmax * per_expert_scale, the
// bucketing of the T*k pairs by rank counting too, and this CTA's job tables.
// Every CTA.
__device__ __noinline__ void topk_phase(const Cfg &P, Smem &S, const moe_layer_w &W) {
    const int T = P.T, E = P.E, k = P.k, n = T * k, H = P.H;
    // the logits as order-preserving unsigned keys (larger logit <=> larger
    // key, exactly): lk[t][e], and their high words kh, in F segments of SL
    // experts per token; a segment takes SS = SL + 4 words (zero padding,
    // below every key), so the F segments that a warp reads at once start in
    // different banks
    unsigned long long *lk = reinterpret_cast<unsigned long long *>(S.pool);  // ring is idle here
    const int F = (E >= 32 && T * E * 4 <= (int)blockDim.x) ? 4 : 1;
    const int SL = ((E + F - 1) / F + 3) & ~3, SS = SL + 4, RS = F * SS;
    uint32_t *kh = reinterpret_cast<uint32_t *>(S.pool + (((size_t)T * E * 8 + 15) & ~(size_t)15));
#pragma unroll 1
    for (int i = threadIdx.x; i < T * RS; i += blockDim.x) {
        const int t = i / RS, r = i - t * RS, q = r / SS, o = r - q * SS, e = q * SL + o;
        uint32_t hi = 0u;
        if (o < SL && e < E) {
            unsigned long long b = (unsigned long long)__double_as_longlong(__ldcg(P.logits + (size_t)t * E + e));
            if (b == 0x8000000000000000ull) b = 0ull;  // -0 and +0 are the same logit
            b = (b >> 63) ? ~b : (b | 0x8000000000000000ull);
            lk[(size_t)t * E + e] = b;
            hi = (uint32_t)(b >> 32);
        }
        kh[i] = hi;
    }
    __syncthreads();
    // rank of (t, e) = keys larger than its key, plus equal keys of lower
    // index.  F adjacent lanes share one (t, e), each counting over one
    // segment of high words: how many are larger and how many equal (its own
    // included).  With no other key sharing its high word, the count of
    // larger high words is the rank; otherwise it is counted again on the
    // full keys.
    const int items = T * E * F;
#pragma unroll 1
    for (int it0 = 0; it0 < items; it0 += blockDim.x) {
        const int it = it0 + threadIdx.x;
        const int te = F == 4 ? it >> 2 : it, f = it - te * F;
        int gt = 0, eq = 0, t = 0, e = 0;
        unsigned long long v = 0ull;
        if (it < items) {
            t = te / E;
            e = te - t * E;
            v = lk[(size_t)t * E + e];
            const uint32_t hv = (uint32_t)(v >> 32);
            const uint4 *seg = reinterpret_cast<const uint4 *>(kh + (size_t)t * RS + f * SS);
#pragma unroll 4
            for (int j = 0; j < SL / 4; ++j) {
                const uint4 h = seg[j];
                gt += (h.x > hv) + (h.y > hv) + (h.z > hv) + (h.w > hv);
                eq += (h.x == hv) + (h.y == hv) + (h.z == hv) + (h.w == hv);
            }
        }
        if (F == 4) {
            gt += __shfl_xor_sync(0xffffffffu, gt, 1);
            gt += __shfl_xor_sync(0xffffffffu, gt, 2);
            eq += __shfl_xor_sync(0xffffffffu, eq, 1);
            eq += __shfl_xor_sync(0xffffffffu, eq, 2);
        }
        if (it < items && f == 0) {
            int rank = gt;
            if (eq > 1) {
                rank = 0;
#pragma unroll 1
                for (int j = 0; j < E; ++j) {
                    const unsigned long long o = lk[(size_t)t * E + j];
                    rank += (o > v) | ((o == v) & (j < e));
                }
            }
            if (rank < k) {
                S.idx[t * k + rank] = e;
                // back from the key to the logit
                const unsigned long long b = (v >> 63) ? (v & 0x7fffffffffffffffull) : ~v;
                S.selv[t * k + rank] = __longlong_as_double((long long)b);
            }
        }
    }
    __syncthreads();
    // bucketing: pair p's position among all pairs ordered by (expert, pair
    // id), and the slot of its expert among the distinct experts (ascending).
    // Few pairs: one pass that also finds first occurrences by rescanning;
    // many pairs: first occurrences in a pass of their own.
    if (T == 1) {
        // one token: its k experts are distinct, so every pair is its expert's
        // only one and the slots are the experts in ascending order
        if (threadIdx.x < n) {
            const int p = threadIdx.x, e = S.idx[p];
            int less = 0;
#pragma unroll 1
            for (int q = 0; q < n; ++q) less += S.idx[q] < e;
            S.perm[less] = p;
            S.tokrow[less] = 0;
            S.act_e[less] = e;
            S.act_off[less] = less;
            S.act_n[less] = 1;
            if (p == 0) S.nact = n;
        }
    } else if (n <= 16) {
        int id[16];  // every pair's expert, in registers
#pragma unroll
        for (int q = 0; q < 16; ++q) id[q] = q < n ? S.idx[q] : 0x7fffffff;
        if (threadIdx.x < n) {
            const int p = threadIdx.x, t = p / k, e = S.idx[p];
            int less = 0, eqb = 0, cnt = 0, slot = 0, nact = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int f = id[q];
                bool firstq = q < n;
#pragma unroll
                for (int r = 0; r < q; ++r) firstq &= id[r] != f;
                less += f < e;
                eqb += (f == e) & (q < p);
                cnt += f == e;
                slot += firstq & (f < e);
                nact += firstq;
            }
            S.perm[less + eqb] = p;
            S.tokrow[less + eqb] = t * H;
            if (eqb == 0) {
                S.act_e[slot] = e;
                S.act_off[slot] = less;
                S.act_n[slot] = cnt;
            }
            if (p == 0) S.nact = nact;
        }
    } else {
        if (threadIdx.x < n) {
            const int p = threadIdx.x, t = p / k, e = S.idx[p];
            int less = 0, eqb = 0, cnt = 0;
#pragma unroll 1
            for (int q = 0; q < n; ++q) {
                const int f = S.idx[q];
                less += f < e;
                eqb += (f == e) & (q < p);
                cnt += f == e;
            }
            S.perm[less + eqb] = p;
            S.tokrow[less + eqb] = t * H;
            S.first[p] = eqb == 0;
            S.poff[p] = less;
            S.pcnt[p] = cnt;
        }
        __syncthreads();
        if (threadIdx.x < n) {
            const int p = threadIdx.x, e = S.idx[p];
            int slot = 0, nact = 0;
#pragma unroll 1
            for (int q = 0; q < n; ++q) {
                slot += S.first[q] & (S.idx[q] < e);
                nact += S.first[q];
            }
            if (S.first[p]) {
                S.act_e[slot] = e;
                S.act_off[slot] = S.poff[p];
                S.act_n[slot] = S.pcnt[p];
            }
            if (p == 0) S.nact = nact;
        }
    }
    if (threadIdx.x < T) S.tokrow_sh[threadIdx.x] = threadIdx.x * H;
    __syncthreads();
    // this layer's gate/up jobs per slot: the shared expert's Is/32, each active slot's I/32
    if ((int)threadIdx.x <= S.nact) S.act_expect[threadIdx.x] += threadIdx.x == 0 ? P.Is / 32 : P.I / 32;
    // task tables of this CTA.  Gate/up jobs are dealt round-robin (every CTA
    // mixes shared-expert jobs with routed ones); down tasks go in contiguous
    // blocks, so that a CTA's tasks share few (slot, part) inputs.
    const int na = S.nact, G = gridDim.x, c = blockIdx.x;
    const int pg = (P.H / 64 + kTaskGroups - 1) / kTaskGroups;
    const int NT2 = (P.Is / 32 + na * (P.I / 32)) * 2 * pg;  // gate/up tasks of the grid
    const int n2 = NT2 > c ? (NT2 - 1 - c) / G + 1 : 0;
    const int RBH = P.H / 32;
    const int J3 = (P.ndp_s + na * P.ndp_r) * RBH;
    const int d0 = (int)((long long)J3 * c / G), d1 = (int)((long long)J3 * (c + 1) / G);
    const int sp0 = d0 / RBH;
    // staged down inputs: the (slot, part) of the CTA's tasks, consecutive; one
    // thread per input, each adding up the sizes of the ones before it
    const int nseg = min(d1 > d0 ? (d1 - 1) / RBH - sp0 + 1 : 0, kMaxSegs);
    const int ngt = min(n2, kMaxTasks), ndt = min(d1 - d0, kMaxTasks);
    if (threadIdx.x < nseg) {
        const int k2 = threadIdx.x;
        int off = 0, slot = 0, part = 0;
#pragma unroll 1
        for (int q = 0; q <= k2; ++q) {
            dn_slot_part(P, sp0 + q, slot, part);
            const int Gs = slot == 0 ? P.Is / 64 : P.I / 64, nd = slot == 0 ? P.ndp_s : P.ndp_r;
            const int ld = (Gs * (part + 1) / nd - Gs * part / nd) * 64;
            const int nn = slot == 0 ? P.T : S.act_n[slot - 1];
            if (q < k2) off += nn * ld;
        }
        const int Gs = slot == 0 ? P.Is / 64 : P.I / 64, nd = slot == 0 ? P.ndp_s : P.ndp_r;
        SegDesc &sg = S.seg[k2];
        sg.slot = (int16_t)slot;
        sg.part = (int16_t)part;
        sg.g0 = (int16_t)(Gs * part / nd);
        sg.ld = (int16_t)((Gs * (part + 1) / nd - sg.g0) * 64);
        sg.n = (int16_t)(slot == 0 ? P.T : S.act_n[slot - 1]);
        sg.seg0 = slot == 0 ? 0 : S.act_off[slot - 1];
        sg.off = off;
        sg.pad = 0;
        if (k2 == nseg - 1) {
            // all inputs at once if they fit the stage (and its chunk sums), else one
            // (slot, part) at a time, each from the start of the stage
            S.seg_rounds = off + sg.n * sg.ld <= min(P.stage_floats, kMaxXs * 32) ? 1 : nseg;
        }
    }
    if (threadIdx.x == 0) {
        S.pg = pg;
        S.ngt = ngt;
        S.ndt = ndt;
        S.nseg = nseg;
        if (nseg == 0) S.seg_rounds = 1;
    }
    // gate/up tables on the first 256 threads, down tables on the rest
    const int half = blockDim.x / 2;
    if ((int)threadIdx.x < half) {
#pragma unroll 1
        for (int i = threadIdx.x; i < ngt; i += half) S.gut[i] = make_gu_task(P, S, c + i * G, pg);
    } else {
#pragma unroll 1
        for (int i = threadIdx.x - half; i < ndt; i += (int)blockDim.x - half) S.dnt[i] = make_dn_task(P, S, d0 + i, sp0);
    }
    __syncthreads();
    if (S.seg_rounds > 1 && (int)threadIdx.x < nseg) S.seg[threadIdx.x].off = 0;
    // the ring was written with generic stores above; order them before the
    // bulk copies (async proxy) that refill it next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
}

// Gate weights w = softmax(logits[top-k]) * per_expert_scale[top-k], in fp64;
// selv[t*k] is token t's largest selected logit.  One warp, off the critical
// path (they are first needed by the combine in the down phase).
__device__ __noinline__ void gate_weights(const Cfg &P, Smem &S, const moe_layer_w &W) {
    const int k = P.k, n = P.T * k;
#pragma unroll 1
    for (int p = threadIdx.x & 31; p < n; p += 32) {
        const int t = p / k;
        const double mx = S.selv[t * k];
        double z = 0.0;
#pragma unroll 1
        for (int s2 = 0; s2 < k; ++s2) z += exp(S.selv[t * k + s2] - mx);
        S.wts[p] = (float)(exp(S.selv[p] - mx) / z * (double)bf16_bits_to_float(W.per_expert_scale[S.idx[p]]));
    }
}

// x' = bf16(rmsnorm_no_scale(h)) pre-scaled for the code decode, and its chunk
// sums, in S.stage.  A thread per 4 columns; the 8 threads of a 32-column
// chunk are adjacent lanes and sum it with three shuffles.
__device__ __noinline__ void stage_x(const Cfg &P, Smem &S) {
    const int T = P.T, H4 = P.H / 4, lane = threadIdx.x & 31;
    const int n4 = T * H4, rounds = (n4 + (int)blockDim.x - 1) / (int)blockDim.x;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {  // every thread runs every round: the shuffles need whole warps
        const int i = r * blockDim.x + threadIdx.x;
        float sx = 0.f;
        if (i < n4) {
            const int t = i / H4;
            float4 v = reinterpret_cast<float4 *>(S.stage)[i];
            const float ri = S.rinv[t];
            const float x0 = bf16_bits_to_float(f32_to_bf16_bits_alu(v.x * ri));
            const float x1 = bf16_bits_to_float(f32_to_bf16_bits_alu(v.y * ri));
            const float x2 = bf16_bits_to_float(f32_to_bf16_bits_alu(v.z * ri));
            const float x3 = bf16_bits_to_float(f32_to_bf16_bits_alu(v.w * ri));
            const int c = (4 * i) & 7;  // 0 or 4
            v.x = x0 * code_prescale(c);
            v.y = x1 * code_prescale(c + 1);
            v.z = x2 * code_prescale(c + 2);
            v.w = x3 * code_prescale(c + 3);
            reinterpret_cast<float4 *>(S.stage)[i] = v;
            sx = (x0 + x1) + (x2 + x3);
        }
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        sx += __shfl_xor_sync(0xffffffffu, sx, 4);
        if (i < n4 && (lane & 7) == 0) S.xs[i >> 3] = sx;
    }
    __syncthreads();
}

// ------------------------------------------------------------------ streaming loops
// (each its own function, so that its register allocation is its own)

// Ring position of task i of a phase that starts at ring sequence number rq.
__device__ __forceinline__ void ring_pos(unsigned rq, int i, int ns, int &s, unsigned &ph) {
    const unsigned q = rq + (unsigned)i;
    s = (int)(q % (unsigned)ns);
    ph = (q / (unsigned)ns) & 1u;
}

// Producer of an expert phase: one ring slot per task, in task order.  The
// ring runs through the gate/up tasks [0, ngt) and on into the down tasks
// [ngt, ngt + ndt) (sequence numbers from the gate/up phase's rq).  In the
// gate/up phase it issues every gate/up task and then the down tasks whose
// slot was last used by a gate/up task (those slots are freed within the
// phase); the down phase issues the rest.  Once the ring is primed, an L2
// prefetch of what comes next (gate/up: the down tasks that do not fit the
// ring; down: this CTA's share of the next layer's shared expert).
__device__ __noinline__ bool task_producer(const Cfg &P, Smem &S, const moe_layer_w &W, bool down, unsigned rq,
                                           const moe_layer_w *next, unsigned &issued) {
    const int ns = P.nslots, ngt = S.ngt, ndt = S.ndt;
    // ring positions [i0, i1) relative to the gate/up phase's first task
    const int pre = min(ndt, ns);  // down tasks issued during the gate/up phase
    const int i0 = down ? ngt + pre : 0, i1 = down ? ngt + ndt : ngt + pre;
    const unsigned rq0 = down ? rq - (unsigned)ngt : rq;
    bool ok = true;
#pragma unroll 1
    for (int i = i0; i < i1; ++i) {
        int s;
        unsigned ph;
        ring_pos(rq0, i, ns, s, ph);
        if (rq0 + (unsigned)i >= (unsigned)ns && !mbar_wait(&S.empty[s], ph ^ 1u, P.err, kErrEmpty)) {
            ok = false;
            break;
        }
        const bool dn = i >= ngt;
        const TaskDesc t = dn ? S.dnt[i - ngt] : S.gut[i];
        const uint32_t *q, *sb;
        task_ptrs(P, W, t, dn, q, sb);
        // the slot now belongs to this task (its previous task has been consumed)
        *reinterpret_cast<volatile unsigned *>(&S.slot_task[s]) = rq0 + (unsigned)i;
        issue_task(S, s, q, sb, t.g0, t.g1);
        issued = rq0 + (unsigned)i + 1u;
        if (!down && i == min(ns, ngt) - 1) {
            // the down tasks beyond the ring: into L2 for now
#pragma unroll 1
            for (int d = pre; d < ndt; ++d) {
                const TaskDesc u = S.dnt[d];
                const uint32_t *uq, *usb;
                task_ptrs(P, W, u, true, uq, usb);
                const int ng = u.g1 - u.g0;
                prefetch_l2(uq + (size_t)u.g0 * 256, (unsigned)ng * kCodeBytesPerGroup);
                prefetch_l2(usb + (size_t)u.g0 * 32, (unsigned)ng * kSbBytesPerGroup);
            }
        }
    }
    if (ok && down && next != nullptr) {
        // this CTA's share of the next layer's shared-expert weights
        const moe_layer_w &N = *next;
        const size_t shq = (size_t)P.Is * P.H / 2, shsb = (size_t)P.Is * (P.H / 64) * 4;
        const void *ptrs[6] = {N.sh_gate.q, N.sh_up.q, N.sh_down.q, N.sh_gate.sb, N.sh_up.sb, N.sh_down.sb};
        const size_t sizes[6] = {shq, shq, shq, shsb, shsb, shsb};
#pragma unroll 1
        for (int a = 0; a < 6; ++a) {
            const size_t per = ((sizes[a] / gridDim.x) + 15) & ~(size_t)15;
            const size_t off = per * blockIdx.x;
            if (off < sizes[a])
                prefetch_range(static_cast<const char *>(ptrs[a]) + off,
                               (off + per <= sizes[a] ? per : sizes[a] - off) & ~(size_t)15);
        }
    }
    return ok;
}

// A team member's share of a task: lanes are the task's 32 rows; acc[tt]
// receives the dot product of the row's groups gi0, gi0 + kWPT, ... (< ng,
// relative to the task's first group) with token tt's input.
template <int NT>
__device__ __forceinline__ void task_dot(const unsigned char *slot, int ng, int gi0, const float *x, const float *xsum,
                                         const int *tokrow, int stride, int n, float (&acc)[NT], int lane) {
#pragma unroll 1
    for (int gi = gi0; gi < ng; gi += kWPT)
        group_dot_n<NT>(slot + gi * kCodeBytesPerGroup,
                        reinterpret_cast<const uint32_t *>(slot + ng * kCodeBytesPerGroup + gi * kSbBytesPerGroup)[lane],
                        x + gi * 64, xsum + 2 * gi, tokrow, stride, n, acc, lane);
}

// A consumer warp's wait for task q in ring slot s: first until the producer
// has handed the slot to q (the slot's previous task is done, so its full
// barrier is in q's phase), then for the phase itself.  Warps take tasks out
// of ring order, so without the first wait a warp could test a phase two
// ahead of the barrier's, which the parity test cannot tell apart.
__device__ __noinline__ bool wait_task(Smem &S, unsigned q, int s, unsigned ph, int *err) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        const volatile unsigned *own = &S.slot_task[s];
        if (*own != q) {
            const unsigned long long t0 = globaltimer();
            while (*own != q) {
                if (globaltimer() - t0 > kWaitNs || ldcg_int(err) != 0) {
                    atomicCAS(err, 0, kErrFull);
                    ok = false;
                    break;
                }
            }
        }
    }
    __syncwarp();
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    return ok && mbar_wait(&S.full[s], ph, err, kErrFull);
}

__device__ __forceinline__ unsigned atom_add_release_gpu(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Bounded wait of one thread until a global count reaches `target` (acquire);
// false (with an error recorded) on a timeout or another CTA's error.
__device__ __noinline__ bool wait_count(const Cfg &P, const unsigned *ctr, unsigned target) {
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 0;; ++it) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
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

template <int NT>
__device__ __noinline__ bool gu_consumer(const Cfg &P, Smem &S, unsigned rq) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, team = wid / kWPT, mb = wid - team * kWPT;
    const int T = P.T, ns = P.nslots, nt = S.ngt, pg = S.pg, pw = pg * kWPT, tpj = 2 * pw;
    bool ok = true;
#pragma unroll 1
    for (int i = team; i < nt; i += kTeams) {
        const TaskDesc t = S.gut[i];
        int s;
        unsigned ph;
        ring_pos(rq, i, ns, s, ph);
        const int n = t.n, ng = t.g1 - t.g0;
        float acc[NT];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) acc[tt] = 0.f;
        const bool got = wait_task(S, rq + (unsigned)i, s, ph, P.err);
        if (got) {
            const int *tokrow = t.slot == 0 ? S.tokrow_sh : S.tokrow + t.seg0;
            const int col = t.g0 * 64;
            task_dot<NT>(S.pool + (size_t)s * kSlotBytes, ng, mb, S.stage + col, S.xs + col / 32, tokrow, 0, n, acc,
                         lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
        if (!got) {
            ok = false;
            continue;
        }
        // this member's partial sums, then its count for the job (release: the
        // warp's stores, ordered by __syncwarp, become visible first)
        float *gp = P.gpart + ((((size_t)t.job * 2 + t.mat) * pg + t.part) * kWPT + mb) * T * 32;
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
            if (tt < n) gp[tt * 32 + lane] = acc[tt];
        __syncwarp();
        unsigned old = 0u;
        if (lane == 0) old = atom_add_release_gpu(&P.cnt_gu[t.job], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (unsigned)(tpj - 1)) {
            // the job's last task: sum the parts in a fixed order, form a = silu(g) * u
            if (lane == 0) __threadfence();
            __syncwarp();
            const float *jp = P.gpart + (size_t)t.job * 2 * pw * T * 32;
#pragma unroll 1
            for (int tt = 0; tt < n; ++tt) {
                float gs = 0.f, us = 0.f;
#pragma unroll
                for (int p2 = 0; p2 < kMaxPG * kWPT; ++p2) {
                    if (p2 < pw) {
                        gs += __ldcg(&jp[((size_t)p2 * T + tt) * 32 + lane]);
                        us += __ldcg(&jp[((size_t)(pw + p2) * T + tt) * 32 + lane]);
                    }
                }
                const float a = silu_mul(gs, us);
                const size_t rs = (size_t)task_rowset(P, t, tt);
                P.act[rs * P.Kmax + t.rb * 32 + lane] = a * code_prescale(lane & 7);
                const float cs = warp_sum(a);  // the job's 32 rows are one 32-column chunk of the down input
                if (lane == 0) P.act_cs[rs * (P.Kmax / 32) + t.rb] = cs;
            }
            __syncwarp();
            if (lane == 0) {
                P.cnt_gu[t.job] = 0u;
                atom_add_release_gpu(&P.act_done[t.slot], 1u);  // the job's rows of a are written
            }
        }
    }
    return ok;
}

// Stage the down inputs of segments [k0, k1): a (already pre-scaled for the
// code decode) and its chunk sums.  Consumer threads only.
__device__ __noinline__ bool stage_segments(const Cfg &P, Smem &S, int k0, int k1) {
    const int ctid = threadIdx.x, KC = P.Kmax / 32;
    // every consumer warp is past its gate/up tasks (the stage still held their
    // input); then wait until each staged slot's SwiGLU rows are all written
    consumer_sync();
    if (ctid == 0) {
        bool ok = true;
        for (int k2 = k0; k2 < k1 && ok; ++k2) ok = wait_count(P, &P.act_done[S.seg[k2].slot], S.act_expect[S.seg[k2].slot]);
        __threadfence();
        S.flag2 = ok;
    }
    consumer_sync();
    if (!S.flag2) return false;
#pragma unroll 1
    for (int k2 = k0; k2 < k1; ++k2) {
        const SegDesc sg = S.seg[k2];
        const int q4 = sg.ld / 4, nc = sg.ld / 32;
        const int rs0 = sg.slot == 0 ? 0 : P.T + sg.seg0;
#pragma unroll 1
        for (int e = ctid; e < sg.n * q4; e += kCWarps * 32) {
            const int tt = e / q4, c4 = e - tt * q4;
            reinterpret_cast<float4 *>(S.stage + sg.off + (size_t)tt * sg.ld)[c4] =
                __ldcg(reinterpret_cast<const float4 *>(P.act + (size_t)(rs0 + tt) * P.Kmax + sg.g0 * 64) + c4);
        }
#pragma unroll 1
        for (int e = ctid; e < sg.n * nc; e += kCWarps * 32) {
            const int tt = e / nc, c = e - tt * nc;
            S.xs[(sg.off + tt * sg.ld) / 32 + c] = __ldcg(&P.act_cs[(size_t)(rs0 + tt) * KC + sg.g0 * 2 + c]);
        }
    }
    consumer_sync();
    return true;
}

// The combine m[t][row] = sum_s w[t,s] * y[t,s] + shared, in a fixed order.
// y and the shared output are sums of kWPT * ndp parts; the loads of up to
// 2 parts x 8 routed slots (or 8 shared parts) are issued before any is used.
__device__ __noinline__ void combine_row(const Cfg &P, const Smem &S, int row) {
    const int T = P.T, k = P.k, H = P.H, ny = P.ndp_r * kWPT, nsh = P.ndp_s * kWPT;
    const size_t ystride = (size_t)T * k * H;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        float mv = 0.f;
#pragma unroll 1
        for (int s0 = 0; s0 < k; s0 += 8) {
            float yv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) yv[u] = 0.f;
#pragma unroll 1
            for (int d0 = 0; d0 < ny; d0 += 2) {
                float pv[2][8];
#pragma unroll
                for (int d = 0; d < 2; ++d)
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        pv[d][u] = (d0 + d < ny && s0 + u < k)
                                       ? __ldcg(&P.y[(d0 + d) * ystride + (size_t)(t * k + s0 + u) * H + row])
                                       : 0.f;
#pragma unroll
                for (int d = 0; d < 2; ++d)
#pragma unroll
                    for (int u = 0; u < 8; ++u) yv[u] += pv[d][u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (s0 + u < k) mv = fmaf(S.wts[t * k + s0 + u], yv[u], mv);
        }
#pragma unroll 1
        for (int u0 = 0; u0 < nsh; u0 += 8) {
            float sv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) sv[u] = u0 + u < nsh ? __ldcg(&P.sh[((size_t)(u0 + u) * T + t) * H + row]) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) mv += sv[u];
        }
        P.m[(size_t)t * H + row] = mv;
    }
}

template <int NT>
__device__ __noinline__ bool dn_consumer(const Cfg &P, Smem &S, unsigned rq) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, team = wid / kWPT, mb = wid - team * kWPT;
    const int T = P.T, k = P.k, H = P.H, ns = P.nslots, nt = S.ndt;
    // member results per row block in this layer: every part of the shared expert and of each active slot
    const unsigned dn_per_rb = (unsigned)((P.ndp_s + S.nact * P.ndp_r) * kWPT);
    const int rounds = S.seg_rounds;
    bool ok = true;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
        const int k0 = rounds == 1 ? 0 : r, k1 = rounds == 1 ? S.nseg : r + 1;
        if (!stage_segments(P, S, k0, k1)) return false;
#pragma unroll 1
        for (int i = team; i < nt; i += kTeams) {
            const TaskDesc t = S.dnt[i];
            if (t.seg < k0 || t.seg >= k1) continue;
            int s;
            unsigned ph;
            ring_pos(rq, i, ns, s, ph);
            const SegDesc sg = S.seg[t.seg];
            const int n = t.n, ng = t.g1 - t.g0;
            float acc[NT];
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) acc[tt] = 0.f;
            const bool got = wait_task(S, rq + (unsigned)i, s, ph, P.err);
            if (got)  // token tt's row at off + tt * ld, its chunk sums at (off + tt * ld) / 32
                task_dot<NT>(S.pool + (size_t)s * kSlotBytes, ng, mb, S.stage + sg.off, S.xs + sg.off / 32, nullptr,
                             sg.ld, n, acc, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[s]);
            if (!got) {
                ok = false;
                continue;
            }
            const int row = t.rb * 32 + lane, pm = t.part * kWPT + mb;
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                if (tt < n) {
                    if (t.slot == 0)
                        P.sh[((size_t)pm * T + tt) * H + row] = acc[tt];
                    else
                        P.y[((size_t)pm * T * k + S.perm[t.seg0 + tt]) * H + row] = acc[tt];
                }
            }
            // count this task for its row block (release: the warp's rows, ordered
            // by __syncwarp, become visible first); the last one forms the combine
            __syncwarp();
            unsigned old = 0u;
            if (lane == 0) old = atom_add_release_gpu(&P.cnt_dn[t.rb], 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == dn_per_rb - 1u) {
                if (lane == 0) __threadfence();
                __syncwarp();
                combine_row(P, S, row);
                __syncwarp();
                if (lane == 0) {
                    P.cnt_dn[t.rb] = 0u;
                    atom_add_release_gpu(P.rows_done, 1u);  // these 32 rows of m are written
                }
            }
        }
        if (rounds > 1) consumer_sync();
    }
    return ok;
}

// All threads: wait until `target` row blocks of m are combined (over all layers so far).
__device__ __noinline__ bool wait_rows(const Cfg &P, Smem &S, unsigned target) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = wait_count(P, P.rows_done, target);
        __threadfence();
        S.flag = ok && ldcg_int(P.err) == 0;
    }
    __syncthreads();
    return S.flag != 0;
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kThreads, 1) decode_stack_kernel(const __grid_constant__ Params Pk) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>(smem_raw);
    const Cfg &P = S.c;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const bool producer = (wid == kProducerWarp && lane == 0);
    const bool consumer = wid < kCWarps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kWPT);  // every warp of the task's team
        }
        mbar_init(&S.rbar, 1);
        for (int s = 0; s < kMaxStages; ++s) S.slot_task[s] = 0xffffffffu;
        for (int s = 0; s <= kMaxPairs; ++s) S.act_expect[s] = 0u;
        S.stage = reinterpret_cast<float *>(S.pool + (size_t)Pk.c.nslots * kSlotBytes);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    copy_words(&S.c, &Pk.c, sizeof(Cfg));
    copy_words(&S.w, &Pk.layers[0], sizeof(moe_layer_w));
    __syncthreads();

    unsigned rq = 0;       // ring sequence number of the next task (the same in every thread)
    unsigned issued = 0;   // producer: tasks whose copies were actually issued
    unsigned rissued = 0;  // producer: router copy batches issued (one per layer)
    unsigned nbar = 0;     // grid barriers passed
    bool ok = true;
    const int ns = P.nslots;

    for (int l = 0; l < P.L && ok; ++l) {
        const moe_layer_w &W = S.w;
        const moe_layer_w *next = l + 1 < P.L ? &Pk.layers[l + 1] : nullptr;
        if (producer) {
            issue_router_copies(P, S, W);
            ++rissued;
        }
        if (l == 0) {
            load_input(P, S, P.h_in);
        } else {
            // every row block of the previous layer's m is combined
            ok = wait_rows(P, S, (unsigned)l * (unsigned)(P.H / 32));
            if (!ok) break;
            finish_layer(P, S, l - 1);
            if (!P.chained) load_input(P, S, P.h_in + (size_t)l * P.T * P.H);
        }
        router_phase(P, S, l);
        ok = grid_sync(P, ++nbar, &S.flag);
        if (!ok) break;
        topk_phase(P, S, W);
        stage_x(P, S);

        // ---------------- gate/up tasks
        if (producer)
            task_producer(P, S, W, false, rq, next, issued);
        else if (consumer) {
            P.T == 1 ? gu_consumer<1>(P, S, rq) : gu_consumer<kMaxT>(P, S, rq);
            if (wid == kCWarps - 1) gate_weights(P, S, W);
        }
        rq += (unsigned)S.ngt;

        // ---------------- down tasks (each CTA as soon as its own gate/up tasks are done)
        if (producer)
            task_producer(P, S, W, true, rq, next, issued);
        else if (consumer)
            P.T == 1 ? dn_consumer<1>(P, S, rq) : dn_consumer<kMaxT>(P, S, rq);
        rq += (unsigned)S.ndt;
        __syncthreads();
        if (threadIdx.x == 0) S.flag = ldcg_int(P.err) == 0;
        if (next != nullptr) copy_words(&S.w, next, sizeof(moe_layer_w));  // every use of this layer's is done
        __syncthreads();
        ok = S.flag != 0;
    }
    if (ok) ok = wait_rows(P, S, (unsigned)P.L * (unsigned)(P.H / 32));
    if (ok) finish_layer(P, S, P.L - 1);  // ok is uniform across the CTA here

    // let this CTA's own bulk copies land before it exits (bounded)
    __syncthreads();
    if (producer) {
        const unsigned first = issued > (unsigned)ns ? issued - ns : 0u;
        for (unsigned q = first; q < issued; ++q) mbar_drain(&S.full[q % ns], (q / ns) & 1);
        if (rissued > 0) mbar_drain(&S.rbar, (rissued - 1) & 1);
    }
}

}  // namespace dec

size_t decode_stack_smem() { return sizeof(dec::Smem); }

static_assert(sizeof(dec::Smem) <= 227 * 1024, "decode kernel shared memory exceeds 227 KiB");
static_assert(sizeof(dec::Params) <= 32000, "decode kernel parameters exceed the 32 KiB limit");
static_assert(sizeof(dec::Cfg) % 4 == 0 && sizeof(moe_layer_w) % 4 == 0, "copied word by word");

struct DecodeWs {
    size_t bar, cnt_dn, cnt_gu, act_done, logits, gpart, act, act_cs, y, sh, m, total, zero_bytes;
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static DecodeWs decode_ws(const moe_layer_w *w, int T) {
    DecodeWs d;
    const int Kmax = w->I > w->Is ? w->I : w->Is;
    const int R = T + T * w->k;
    const int ndp_r = (w->I / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    const int ndp_s = (w->Is / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += al256(b);
        return o;
    };
    d.bar = take(256);
    const size_t pairs = (size_t)T * w->k < (size_t)w->E ? (size_t)T * w->k : (size_t)w->E;
    const size_t jobs = (size_t)w->Is / 32 + pairs * (w->I / 32);
    const size_t pg = (w->H / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    d.cnt_dn = take(sizeof(unsigned) * (size_t)(w->H / 32));
    d.cnt_gu = take(sizeof(unsigned) * jobs);
    d.act_done = take(sizeof(unsigned) * (R + 1));  // per slot, then rows_done
    d.zero_bytes = off;
    d.gpart = take(sizeof(float) * jobs * 2 * pg * dec::kWPT * T * 32);
    d.logits = take(sizeof(double) * (size_t)T * w->E);
    d.act = take(sizeof(float) * (size_t)R * Kmax);
    d.act_cs = take(sizeof(float) * (size_t)R * (Kmax / 32));
    d.y = take(sizeof(float) * (size_t)ndp_r * dec::kWPT * T * w->k * w->H);
    d.sh = take(sizeof(float) * (size_t)ndp_s * dec::kWPT * T * w->H);
    d.m = take(sizeof(float) * (size_t)T * w->H);
    d.total = off;
    return d;
}

size_t decode_stack_ws_bytes(const moe_layer_w *w, int T) { return decode_ws(w, T).total; }

size_t decode_stack_status_offset() { return sizeof(unsigned); }

// Split of the shared-memory pool between the ring and the input stage for
// calls of T tokens on layers shaped like w; false if the shape does not fit.
static bool decode_layout(const moe_layer_w &w, int T, int grid, int *nslots, int *stage_floats) {
    const long th = (long)T * w.H, tdn = (long)T * dec::kTaskGroups * 64;
    long stage = th > tdn ? th : tdn;
    if (stage > dec::kStageFloats || stage / 32 > dec::kMaxXs) return false;
    stage = (stage + 31) & ~31L;  // keep the stage 128-byte aligned
    long ns = (dec::kPoolBytes - stage * 4) / dec::kSlotBytes;
    if (ns > dec::kMaxStages) ns = dec::kMaxStages;
    const long ring = ns * dec::kSlotBytes;
    const long rows = grid > 0 ? (w.E + grid - 1) / grid : w.E;
    const long rcopy = 2L * w.H + rows * w.H + 2 * (rows * (w.H / 64) * 2 + 32);
    const long topk_keys = (long)T * w.E * 8 + 16 + (long)T * (w.E + 28) * 4;  // keys and padded high words
    if (ns < 3 || topk_keys > ring || rcopy > ring || grid <= 0) return false;
    // task tables of the busiest CTA, for the most distinct experts a call can route to
    const long pairs = (long)T * w.k < w.E ? (long)T * w.k : w.E;
    const long pg = (w.H / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    const long j2 = w.Is / 32 + pairs * (w.I / 32);
    const long ndp_r = (w.I / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    const long ndp_s = (w.Is / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    const long rbh = w.H / 32, j3 = (ndp_s + pairs * ndp_r) * rbh;
    const long gu_tasks = (j2 * 2 * pg + grid - 1) / grid, dn_tasks = (j3 + grid - 1) / grid;
    if (pg > dec::kMaxPG || gu_tasks > dec::kMaxTasks || dn_tasks > dec::kMaxTasks ||
        (dn_tasks + rbh - 1) / rbh + 1 > dec::kMaxSegs)
        return false;
    *nslots = (int)ns;
    *stage_floats = (int)((dec::kPoolBytes - ring) / 4);
    return true;
}

bool decode_stack_fits(const moe_layer_w *w, int T, int grid) {
    int a, b;
    return decode_layout(*w, T, grid, &a, &b);
}

int decode_stack_max_tokens() { return dec::kMaxT; }
int decode_stack_max_layers() { return dec::kMaxLayers; }
int decode_stack_stage_floats() { return dec::kStageFloats; }

cudaError_t launch_decode_stack(const moe_layer_w *layers, int L, const uint16_t *h_in, int chained,
                                uint16_t *h_out, int T, void *ws, const moe_opts &o, int grid, cudaStream_t st) {
    const moe_layer_w &w = layers[0];
    const DecodeWs d = decode_ws(&w, T);
    dec::Params Pk;  // ~10 KiB, passed by value (kernel parameters up to 32 KiB)
    dec::Cfg &P = Pk.c;
    for (int l = 0; l < L; ++l) Pk.layers[l] = layers[l];
    P.h_in = h_in;
    P.h_out = h_out;
    P.L = L;
    P.T = T;
    P.chained = chained;
    P.post_norm = o.post_norm;
    P.layer_scalar = o.layer_scalar;
    P.eps = o.eps;
    P.H = w.H;
    P.E = w.E;
    P.k = w.k;
    P.I = w.I;
    P.Is = w.Is;
    P.Kmax = w.I > w.Is ? w.I : w.Is;
    P.R = T + T * w.k;
    P.ndp_r = (w.I / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    P.ndp_s = (w.Is / 64 + dec::kTaskGroups - 1) / dec::kTaskGroups;
    if (!decode_layout(w, T, grid, &P.nslots, &P.stage_floats)) return cudaErrorInvalidValue;
    char *base = static_cast<char *>(ws);
    P.bar = reinterpret_cast<unsigned *>(base + d.bar);
    // test hook: MOE_TEST_BARRIER_EXTRA=1 makes the first grid barrier wait for an
    // arrival that never comes, so that its bounded wait runs out (about 1 s) and
    // the kernel reports "grid barrier timed out" through the workspace status
    const char *extra = getenv("MOE_TEST_BARRIER_EXTRA");
    P.bar_extra = (extra && extra[0] == '1') ? 1u : 0u;
    P.err = reinterpret_cast<int *>(base + d.bar + sizeof(unsigned));
    P.logits = reinterpret_cast<double *>(base + d.logits);
    P.cnt_dn = reinterpret_cast<unsigned *>(base + d.cnt_dn);
    P.cnt_gu = reinterpret_cast<unsigned *>(base + d.cnt_gu);
    P.act_done = reinterpret_cast<unsigned *>(base + d.act_done);
    P.rows_done = P.act_done + (T + T * w.k);
    P.gpart = reinterpret_cast<float *>(base + d.gpart);
    P.act = reinterpret_cast<float *>(base + d.act);
    P.act_cs = reinterpret_cast<float *>(base + d.act_cs);
    P.y = reinterpret_cast<float *>(base + d.y);
    P.sh = reinterpret_cast<float *>(base + d.sh);
    P.m = reinterpret_cast<float *>(base + d.m);

    const size_t smem = sizeof(dec::Smem);
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(dec::decode_stack_kernel), smem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ws, 0, d.zero_bytes, st);
    if (e != cudaSuccess) return e;
    void *args[] = {&Pk};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(dec::decode_stack_kernel), dim3(grid),
                                    dim3(dec::kThreads), args, smem, st);
    return e;
}

cudaError_t decode_stack_grid(int device, int *grid) {
    int sms = 0, per = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) return e;
    e = ensure_smem(reinterpret_cast<const void *>(dec::decode_stack_kernel), sizeof(dec::Smem));
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, dec::decode_stack_kernel, dec::kThreads,
                                                      sizeof(dec::Smem));
    if (e != cudaSuccess) return e;
    *grid = per >= 1 ? sms : 0;
    return cudaSuccess;
}

}  // namespace moe
