// moe_wsmma.cu -- the expert FFN of a batch of tokens on the warp-level
// tensor cores, weight-stationary: every weight of a 32-row block is read
// once per group of tokens and multiplied against up to 8 (gate/up) or 16
// (down) tokens at a time.
//
// TurboFieldfare introduction page (discuss.pytorch.kr), section
// "TurboFieldfare's expert streaming structure": prefill runs in chunks of up
// to 128 tokens so that one read of an expert serves every row routed to it;
// section "How TurboFieldfare saves memory": MLX affine 4-bit weights in
// groups of 64 with a BF16 scale and bias.  After bucketing, an expert sees
// few rows (a 128-token chunk gives ~8 per expert), so its FFN is a small
// matrix product whose cost is the weight bytes, not the FLOPs.
//
// Operands (m16n8k16, FP16 inputs, FP32 accumulation):
//   codes   a nibble q masked in place into the low bits of an FP16 half is
//           the subnormal q * 2^-24, exact; one mask per pair of nibbles
//           (j, j+4) of a word, and no offset that would cancel later.  The
//           odd nibbles (1,5), (3,7) are masked at bits 4..7 of each half,
//           where they read 16 q * 2^-24 (still subnormal and exact), so a
//           word takes one shift (by 8) and four masks;
//   inputs  the gathered token rows (FP16, every 8 columns stored in the
//           order 0,4,1,5,2,6,3,7, as the tcgen05 path stores them), so one
//           16-byte load gives a lane the values of one code word in the
//           MMA's K order.  The odd columns hold x / 16 (the gather and the
//           gate/up epilogue round x / 16 once), so every product is
//           q * 2^-24 * x, exact while x / 16 is an FP16 normal (|x| >= 2^-10);
//   group of 64 columns:  sum_k (s q_k + b) x_k = (s 2^24) D + b sum_k x_k,
//           D = sum_k (q_k 2^-24) x_k, with sum_k x_k from MMAs against ones
//           (16 against the odd columns).
// The scale and bias stay FP32, so only the token rows and the SwiGLU values
// are FP16 here; a SwiGLU value beyond the FP16 range is recorded in the
// range status word (and stored as 0), as on the tcgen05 path.
//
// Work items: (row blocks, token group) of the shared expert, then of every
// active routed expert; a persistent grid of 4 CTAs of 4 warps per SM walks
// them.  Every sum is taken in a fixed order, so results do not depend on
// timing.
//   gate/up  one 32-row block and 8 tokens: the 4 warps split the 64-column
//            groups of K and add their partial sums in shared memory in warp
//            order.  A = 8 gate rows (M 0..7) and the same 8 up rows (M 8..15)
//            of one of the block's four 8-row slices, B = 8 tokens; the SwiGLU
//            output goes to the FP16 activation buffer (the down GEMM's input,
//            in the same 8-column order).
//   down     four 32-row blocks and 16 tokens: warp w owns block w over all
//            of K, so its sums are the outputs (a shared-expert item is one
//            block whose K the 4 warps split, summed in shared memory in warp
//            order).  A = 16 tokens' activations,
//            B = 8 rows of one slice; the output goes to y (routed, by pair
//            id) or sh (shared, by token).
#include <cuda_fp16.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace wsm {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = 4;             // 16 warps of 128 registers per SM
constexpr int kMaxSlots = 1024;           // active experts a call may have (E <= 1024)
constexpr uint32_t kOnes = 0x3C003C00u;   // FP16 pair (1, 1)
constexpr uint32_t kSixteens = 0x4C004C00u;  // FP16 pair (16, 16): the weight of an odd column's x / 16
constexpr float kCodeScale = 16777216.f;  // 2^24: undoes the subnormal code encoding

struct Params {
    const uint32_t *q[2], *sb[2];    // routed matrices (tiled, stacked over experts): gate, up / down
    const uint32_t *sq[2], *ssb[2];  // the shared expert's
    int rows_r, rows_s;              // output rows of a routed / the shared matrix
    int K_r, K_s;                    // input columns
    int T, with_shared, ntok;        // ntok: tokens per item (8 gate/up, 16 down)
    const int32_t *offsets, *perm, *active;
    const uint16_t *xin;  // FP16 input rows [T + T*k, ld_in]
    int ld_in;
    uint16_t *act;  // gate/up output [T + T*k, act_ld] FP16
    int act_ld;
    float *y, *sh;  // down outputs: routed [T*k, H] by pair id, shared [T, H]
    int H;
    int *range_err;
};

struct Item {
    bool shared;
    int e, rb, row0, n;  // expert, row block, first token row in xin/act, tokens in this item (1..ntok)
    int seg;             // first bucket position of the item (routed) or first token (shared)
};

// cum[s] = token groups of the active slots before s; cum[na] = all of them.
__device__ int build_prefix(const Params &P, int *cum) {
    __shared__ int wsum[kWarps];
    const int na = __ldg(P.active);
    constexpr int kPer = kMaxSlots / kThreads;
    const int per = (na + kThreads - 1) / kThreads;  // slots per thread (<= kPer)
    const int s0 = threadIdx.x * per;
    int loc[kPer], tot = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        loc[i] = 0;
        if (i < per && s0 + i < na) {
            const int e = __ldg(P.active + 1 + s0 + i);
            const int n = __ldg(P.offsets + e + 1) - __ldg(P.offsets + e);
            loc[i] = (n + P.ntok - 1) / P.ntok;
        }
        tot += loc[i];
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int run = base + inc - tot;
    for (int i = 0; i < per; ++i)
        if (s0 + i < na) {
            cum[s0 + i] = run;
            run += loc[i];
        }
    int all = 0;
    for (int w = 0; w < kWarps; ++w) all += wsum[w];
    if (threadIdx.x == 0) cum[na] = all;
    __syncthreads();
    return all;
}

__device__ __forceinline__ Item get_item(const Params &P, const int *cum, int na, int id, int nsh, int rbs_s,
                                         int rbs_r) {
    Item it;
    if (id < nsh) {
        const int tg = id / rbs_s;
        it.shared = true;
        it.e = 0;
        it.rb = id - tg * rbs_s;
        it.seg = tg * P.ntok;
        it.row0 = it.seg;
        it.n = min(P.ntok, P.T - it.seg);
        return it;
    }
    id -= nsh;
    const int u = id / rbs_r;
    it.shared = false;
    it.rb = id - u * rbs_r;
    int lo = 0, hi = na;  // the last s with cum[s] <= u
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= u) lo = mid;
        else hi = mid;
    }
    it.e = __ldg(P.active + 1 + lo);
    const int first = __ldg(P.offsets + it.e), cnt = __ldg(P.offsets + it.e + 1) - first;
    const int tg = u - cum[lo];
    it.seg = first + tg * P.ntok;
    it.row0 = P.T + it.seg;
    it.n = min(P.ntok, cnt - tg * P.ntok);
    return it;
}

// Nibble pairs (0,4), (1,5), (2,6), (3,7) of a code word as FP16 pairs: q * 2^-24 for the even
// nibbles, 16 q * 2^-24 for the odd ones (their inputs are stored divided by 16).
__device__ __forceinline__ void code_pairs(uint32_t w, uint32_t (&p)[4]) {
    constexpr uint32_t kM = 0x000F000Fu, kM4 = 0x00F000F0u;
    const uint32_t w8 = w >> 8;
    p[0] = w & kM;
    p[1] = w & kM4;
    p[2] = w8 & kM;
    p[3] = w8 & kM4;
}

__device__ __forceinline__ void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                    uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 ldg_v2(const uint32_t *p) { return __ldg(reinterpret_cast<const uint2 *>(p)); }
__device__ __forceinline__ uint4 ldg_v4(const uint16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// One group of 64 columns of a gate/up item as a lane holds it: for slice s,
// words 2(t&1), 2(t&1)+1 of chunk 2gi + (t>>1) of gate row s*8+g (cg) and of
// up row s*8+g (cu); the token's 16 matching input values (x0, x1); the two
// rows' (scale, bias) words.
struct GUStage {
    uint2 cg[4], cu[4];
    uint4 x0, x1;
    uint32_t sg[4], su[4];
};

struct GUView {
    const uint32_t *qg, *qu, *sbg, *sbu;  // this lane's words / row in slice 0, group 0
    const uint16_t *x;                    // this lane's token row, at its words' columns of group 0
    bool xok;
};

__device__ __forceinline__ void gu_load(const GUView &v, int gi, GUStage &s) {
    // a group is 2 chunks = 256 code words of the row block, 32 (scale, bias) words
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
        s.cg[sl] = ldg_v2(v.qg + (size_t)gi * 256 + sl * 32);
        s.cu[sl] = ldg_v2(v.qu + (size_t)gi * 256 + sl * 32);
        s.sg[sl] = __ldg(v.sbg + (size_t)gi * 32 + sl * 8);
        s.su[sl] = __ldg(v.sbu + (size_t)gi * 32 + sl * 8);
    }
    if (v.xok) {
        s.x0 = ldg_v4(v.x + gi * 64);
        s.x1 = ldg_v4(v.x + gi * 64 + 8);
    } else {
        s.x0 = s.x1 = make_uint4(0u, 0u, 0u, 0u);
    }
}

__device__ __forceinline__ void gu_compute(const GUStage &s, float (&acc)[4][4]) {
    float dx[4] = {0.f, 0.f, 0.f, 0.f};
    mma(dx, kOnes, kOnes, kSixteens, kSixteens, s.x0.x, s.x0.y);
    mma(dx, kOnes, kOnes, kSixteens, kSixteens, s.x0.z, s.x0.w);
    mma(dx, kOnes, kOnes, kSixteens, kSixteens, s.x1.x, s.x1.y);
    mma(dx, kOnes, kOnes, kSixteens, kSixteens, s.x1.z, s.x1.w);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t g0[4], g1[4], u0[4], u1[4];
        code_pairs(s.cg[sl].x, g0);
        code_pairs(s.cg[sl].y, g1);
        code_pairs(s.cu[sl].x, u0);
        code_pairs(s.cu[sl].y, u1);
        mma(d, g0[0], u0[0], g0[1], u0[1], s.x0.x, s.x0.y);
        mma(d, g0[2], u0[2], g0[3], u0[3], s.x0.z, s.x0.w);
        mma(d, g1[0], u1[0], g1[1], u1[1], s.x1.x, s.x1.y);
        mma(d, g1[2], u1[2], g1[3], u1[3], s.x1.z, s.x1.w);
        const float sg = bf16_bits_to_float(s.sg[sl] & 0xffffu) * kCodeScale, bg = bf16_bits_to_float(s.sg[sl] >> 16);
        const float su = bf16_bits_to_float(s.su[sl] & 0xffffu) * kCodeScale, bu = bf16_bits_to_float(s.su[sl] >> 16);
        acc[sl][0] = fmaf(sg, d[0], fmaf(bg, dx[0], acc[sl][0]));
        acc[sl][1] = fmaf(sg, d[1], fmaf(bg, dx[1], acc[sl][1]));
        acc[sl][2] = fmaf(su, d[2], fmaf(bu, dx[0], acc[sl][2]));
        acc[sl][3] = fmaf(su, d[3], fmaf(bu, dx[1], acc[sl][3]));
    }
}

__device__ __forceinline__ GUView gu_view(const Params &P, const Item &it, int lane) {
    const int g = lane >> 2, t = lane & 3, G = P.H / 64, C = P.H / 32;
    const int rows = it.shared ? P.rows_s : P.rows_r;
    const size_t mrb = it.shared ? (size_t)it.rb : (size_t)it.e * (rows / 32) + it.rb;
    // this lane's codes: chunk (t>>1) of group 0, row g of slice 0, words 2(t&1) and 2(t&1)+1
    const size_t qoff = (mrb * C + (t >> 1)) * 128 + g * 4 + 2 * (t & 1);
    GUView v;
    v.qg = (it.shared ? P.sq[0] : P.q[0]) + qoff;
    v.qu = (it.shared ? P.sq[1] : P.q[1]) + qoff;
    v.sbg = (it.shared ? P.ssb[0] : P.sb[0]) + mrb * G * 32 + g;
    v.sbu = (it.shared ? P.ssb[1] : P.sb[1]) + mrb * G * 32 + g;
    v.xok = g < it.n;
    v.x = P.xin + (size_t)(it.row0 + (v.xok ? g : 0)) * P.ld_in + (t >> 1) * 32 + 16 * (t & 1);
    return v;
}

// Items are software-pipelined: the first K group of a warp's next item is loaded before the
// current item's partial sums meet in shared memory, so the item's first HBM latency overlaps them.
__global__ void __launch_bounds__(kThreads, kCtasPerSm) gateup_kernel(const Params P) {
    __shared__ int cum[kMaxSlots + 1];
    __shared__ float red[kWarps][16][32];
    const int na = __ldg(P.active);
    const int units = build_prefix(P, cum);
    const int rbs_s = P.rows_s / 32, rbs_r = P.rows_r / 32;
    const int nsh = P.with_shared ? rbs_s * ((P.T + P.ntok - 1) / P.ntok) : 0;
    const int total = nsh + units * rbs_r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int G = P.H / 64;
    Item it;
    GUView v;
    GUStage cur;
    if (blockIdx.x < total) {
        it = get_item(P, cum, na, blockIdx.x, nsh, rbs_s, rbs_r);
        v = gu_view(P, it, lane);
        if (warp < G) gu_load(v, warp, cur);
    }
    for (int id = blockIdx.x; id < total; id += gridDim.x) {
        float acc[4][4];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) acc[sl][0] = acc[sl][1] = acc[sl][2] = acc[sl][3] = 0.f;
        int gi = warp;
        if (gi < G) {
            GUStage nxt;
            for (; gi + kWarps < G; gi += kWarps) {
                gu_load(v, gi + kWarps, nxt);
                gu_compute(cur, acc);
                cur = nxt;
            }
            gu_compute(cur, acc);
        }
        const Item ic = it;  // this item; `it`, `v` and `cur` move on to the next one
        if (id + (int)gridDim.x < total) {
            it = get_item(P, cum, na, id + gridDim.x, nsh, rbs_s, rbs_r);
            v = gu_view(P, it, lane);
            if (warp < G) gu_load(v, warp, cur);
        }
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
#pragma unroll
            for (int c = 0; c < 4; ++c) red[warp][sl * 4 + c][lane] = acc[sl][c];
        __syncthreads();
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            // warp w: slice w, token columns 2t and 2t + 1
            const int sl = warp;
            float gs = 0.f, us = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                gs += red[w][sl * 4 + h][lane];
                us += red[w][sl * 4 + 2 + h][lane];
            }
            const int j = 2 * t + h;
            if (j < ic.n) {
                const int r = ic.rb * 32 + sl * 8 + g;  // gate/up row = activation column
                const int col = (r & ~7) | ((r & 3) << 1) | ((r >> 2) & 1);
                float a = silu_mul(gs, us);
                if (!(fabsf(a) <= 65504.f)) {
                    atomicCAS(P.range_err, 0, 2);
                    a = 0.f;
                }
                if (r & 1) a *= 0.0625f;  // an odd column of the down GEMM's input: a / 16
                P.act[(size_t)(ic.row0 + j) * P.act_ld + col] = __half_as_ushort(__float2half_rn(a));
            }
        }
        __syncthreads();
    }
}

// One group of a down item as a lane holds it: for slice s, words 2(t&1),
// 2(t&1)+1 of chunk 2gi + (t>>1) of row s*8+g (the B operand's column g); the
// two tokens' 16 matching activations each; the (scale, bias) words of rows
// s*8+2t and s*8+2t+1 (this lane's D columns).
struct DStage {
    uint2 c[4];
    uint4 a00, a01, a10, a11;  // token j0: its two words' values; token j1: the same
    uint2 sb[4];
};

struct DView {
    const uint32_t *q, *sb;
    const uint16_t *a0, *a1;
    bool ok0, ok1;
};

__device__ __forceinline__ void d_load(const DView &v, int gi, DStage &s) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
        s.c[sl] = ldg_v2(v.q + (size_t)gi * 256 + sl * 32);
        s.sb[sl] = ldg_v2(v.sb + (size_t)gi * 32 + sl * 8);
    }
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    s.a00 = v.ok0 ? ldg_v4(v.a0 + gi * 64) : z;
    s.a01 = v.ok0 ? ldg_v4(v.a0 + gi * 64 + 8) : z;
    s.a10 = v.ok1 ? ldg_v4(v.a1 + gi * 64) : z;
    s.a11 = v.ok1 ? ldg_v4(v.a1 + gi * 64 + 8) : z;
}

__device__ __forceinline__ void d_compute(const DStage &s, float (&y)[4][4]) {
    float da[4] = {0.f, 0.f, 0.f, 0.f};
    mma(da, s.a00.x, s.a10.x, s.a00.y, s.a10.y, kOnes, kSixteens);
    mma(da, s.a00.z, s.a10.z, s.a00.w, s.a10.w, kOnes, kSixteens);
    mma(da, s.a01.x, s.a11.x, s.a01.y, s.a11.y, kOnes, kSixteens);
    mma(da, s.a01.z, s.a11.z, s.a01.w, s.a11.w, kOnes, kSixteens);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t p0[4], p1[4];
        code_pairs(s.c[sl].x, p0);
        code_pairs(s.c[sl].y, p1);
        mma(d, s.a00.x, s.a10.x, s.a00.y, s.a10.y, p0[0], p0[1]);
        mma(d, s.a00.z, s.a10.z, s.a00.w, s.a10.w, p0[2], p0[3]);
        mma(d, s.a01.x, s.a11.x, s.a01.y, s.a11.y, p1[0], p1[1]);
        mma(d, s.a01.z, s.a11.z, s.a01.w, s.a11.w, p1[2], p1[3]);
        const float s0 = bf16_bits_to_float(s.sb[sl].x & 0xffffu) * kCodeScale, b0 = bf16_bits_to_float(s.sb[sl].x >> 16);
        const float s1 = bf16_bits_to_float(s.sb[sl].y & 0xffffu) * kCodeScale, b1 = bf16_bits_to_float(s.sb[sl].y >> 16);
        // d: [j0][row 2t], [j0][2t+1], [j1][2t], [j1][2t+1]; da[0], da[2]: the two tokens' input sums
        y[sl][0] = fmaf(s0, d[0], fmaf(b0, da[0], y[sl][0]));
        y[sl][1] = fmaf(s1, d[1], fmaf(b1, da[0], y[sl][1]));
        y[sl][2] = fmaf(s0, d[2], fmaf(b0, da[2], y[sl][2]));
        y[sl][3] = fmaf(s1, d[3], fmaf(b1, da[2], y[sl][3]));
    }
}

// Routed down items are 4 row blocks (128 output rows) of one expert and 16 tokens: warp w owns row
// block 4*ib + w over all of K (I columns), so its sums are the outputs.  The shared expert's K (Is
// columns) is usually several times longer, so its items are one row block whose K groups the 4 warps
// split, adding their sums in shared memory in warp order: every item then takes about as long, and
// the round-robin over items stays balanced.
constexpr int kDownRbs = kWarps;

// A warp's part of a down item: its row block, whether the block exists, the K groups, the view.
struct DWork {
    int rb, G, gi0, step;  // row block; K groups; this warp's first group and group stride
    bool live;
    DView v;
};

__device__ __forceinline__ DWork d_work(const Params &P, const Item &it, int warp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int K = it.shared ? P.K_s : P.K_r, C = K / 32, rows = it.shared ? P.rows_s : P.rows_r;
    DWork w;
    w.G = K / 64;
    w.rb = it.shared ? it.rb : it.rb * kDownRbs + warp;  // this warp's row block
    w.gi0 = it.shared ? warp : 0;
    w.step = it.shared ? kWarps : 1;
    w.live = w.rb < rows / 32 && w.gi0 < w.G;
    const size_t mrb = it.shared ? (size_t)w.rb : (size_t)it.e * (rows / 32) + w.rb;
    w.v.q = (it.shared ? P.sq[0] : P.q[0]) + (mrb * C + (t >> 1)) * 128 + g * 4 + 2 * (t & 1);
    w.v.sb = (it.shared ? P.ssb[0] : P.sb[0]) + mrb * w.G * 32 + 2 * t;
    w.v.ok0 = g < it.n;
    w.v.ok1 = g + 8 < it.n;
    const int xo = (t >> 1) * 32 + 16 * (t & 1);
    w.v.a0 = P.xin + (size_t)(it.row0 + (w.v.ok0 ? g : 0)) * P.ld_in + xo;
    w.v.a1 = P.xin + (size_t)(it.row0 + (w.v.ok1 ? g + 8 : 0)) * P.ld_in + xo;
    return w;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm) down_kernel(const Params P) {
    __shared__ int cum[kMaxSlots + 1];
    __shared__ float red[kWarps][16][32];
    const int na = __ldg(P.active);
    const int units = build_prefix(P, cum);
    // items per token tile: shared, one row block each; routed, the row blocks in runs of kDownRbs
    const int rbs_s = P.rows_s / 32, rbs_r = (P.rows_r / 32 + kDownRbs - 1) / kDownRbs;
    const int nsh = P.with_shared ? rbs_s * ((P.T + P.ntok - 1) / P.ntok) : 0;
    const int total = nsh + units * rbs_r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    // software-pipelined over items like gateup_kernel
    Item it;
    DWork dw;
    DStage cur;
    if (blockIdx.x < total) {
        it = get_item(P, cum, na, blockIdx.x, nsh, rbs_s, rbs_r);  // it.rb: the run of row blocks
        dw = d_work(P, it, warp, lane);
        if (dw.live) d_load(dw.v, dw.gi0, cur);
    }
    for (int id = blockIdx.x; id < total; id += gridDim.x) {
        float y[4][4];
#pragma unroll
        for (int sl = 0; sl < 4; ++sl) y[sl][0] = y[sl][1] = y[sl][2] = y[sl][3] = 0.f;
        if (dw.live) {
            DStage nxt;
            int gi = dw.gi0;
            for (; gi + dw.step < dw.G; gi += dw.step) {
                d_load(dw.v, gi + dw.step, nxt);
                d_compute(cur, y);
                cur = nxt;
            }
            d_compute(cur, y);
        }
        const Item ic = it;  // this item; `it`, `dw` and `cur` move on to the next one
        const int rb = dw.rb;
        const bool live = dw.live;
        if (id + (int)gridDim.x < total) {
            it = get_item(P, cum, na, id + gridDim.x, nsh, rbs_s, rbs_r);
            dw = d_work(P, it, warp, lane);
            if (dw.live) d_load(dw.v, dw.gi0, cur);
        }
        if (ic.shared) {
            // the 4 warps' partial sums of row block rb; warp w writes slice w
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
#pragma unroll
                for (int c = 0; c < 4; ++c) red[warp][sl * 4 + c][lane] = y[sl][c];
            __syncthreads();
            if (rb < P.rows_s / 32) {
                const int sl = warp;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = g + 8 * h;
                    float o0 = 0.f, o1 = 0.f;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) {
                        o0 += red[w][sl * 4 + 2 * h][lane];
                        o1 += red[w][sl * 4 + 2 * h + 1][lane];
                    }
                    if (j < ic.n)
                        *reinterpret_cast<float2 *>(P.sh + (size_t)(ic.seg + j) * P.H + rb * 32 + sl * 8 + 2 * t) =
                            make_float2(o0, o1);
                }
            }
            __syncthreads();
        } else if (live) {
            // y[sl]: token g (0, 1) and token g + 8 (2, 3), rows 2t and 2t + 1 of slice sl of row block rb
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = g + 8 * h;
                if (j < ic.n) {
                    float *dst = P.y + (size_t)__ldg(P.perm + ic.seg + j) * P.H;
#pragma unroll
                    for (int sl = 0; sl < 4; ++sl)
                        *reinterpret_cast<float2 *>(dst + rb * 32 + sl * 8 + 2 * t) =
                            make_float2(y[sl][2 * h], y[sl][2 * h + 1]);
                }
            }
        }
    }
}

// SM count of the device that runs launches on `st`.
int sms_of(cudaStream_t st) {
    int dev = 0, n = 0;
    if (stream_device(st, &dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace wsm

bool wsmma_supported(const moe_layer_w *w) { return w->E <= wsm::kMaxSlots; }

cudaError_t launch_expert_wsmma(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                                const int32_t *perm, const int32_t *active, int with_shared, const MmaBuffers &b,
                                cudaStream_t st) {
    using namespace wsm;
    if (!wsmma_supported(w)) return cudaErrorInvalidValue;
    const int H = w->H, k = w->k, I = w->I, Is = w->Is;
    const int Kmax = I > Is ? I : Is;
    cudaError_t e = launch_gather_tokens(xe, perm, T, k, H, b.xg, st, true);
    if (e != cudaSuccess) return e;
    const int sms = sms_of(st);
    if (sms <= 0) return cudaErrorNoDevice;
    const long long pairs = (long long)T * k;
    const long long max_active = pairs < w->E ? pairs : w->E;
    Params P{};
    P.T = T;
    P.with_shared = with_shared;
    P.offsets = offsets;
    P.perm = perm;
    P.active = active;
    P.act = b.act;
    P.act_ld = Kmax;
    P.y = b.y;
    P.sh = b.sh;
    P.H = H;
    P.range_err = b.range_err;

    // gate/up: items of 8 tokens; an active expert has at most n_e/8 + 1 groups of them
    P.q[0] = w->gate.q;
    P.sb[0] = w->gate.sb;
    P.q[1] = w->up.q;
    P.sb[1] = w->up.sb;
    P.sq[0] = w->sh_gate.q;
    P.ssb[0] = w->sh_gate.sb;
    P.sq[1] = w->sh_up.q;
    P.ssb[1] = w->sh_up.sb;
    P.rows_r = I;
    P.rows_s = Is;
    P.K_r = P.K_s = H;
    P.xin = b.xg;
    P.ld_in = H;
    P.ntok = 8;
    long long items =
        (with_shared ? (long long)(Is / 32) * ((T + 7) / 8) : 0) + (pairs / 8 + max_active) * (I / 32);
    int grid = (int)(items < (long long)kCtasPerSm * sms ? items : (long long)kCtasPerSm * sms);
    if (grid > 0) {
        gateup_kernel<<<grid, kThreads, 0, st>>>(P);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // down: items of 16 tokens
    P.q[0] = w->down.q;
    P.sb[0] = w->down.sb;
    P.q[1] = P.sb[1] = nullptr;
    P.sq[0] = w->sh_down.q;
    P.ssb[0] = w->sh_down.sb;
    P.sq[1] = P.ssb[1] = nullptr;
    P.rows_r = P.rows_s = H;
    P.K_r = I;
    P.K_s = Is;
    P.xin = b.act;
    P.ld_in = Kmax;
    P.ntok = 16;
    const long long drun = (H / 32 + kDownRbs - 1) / kDownRbs;
    items = (with_shared ? (long long)(H / 32) * ((T + 15) / 16) : 0) + (pairs / 16 + max_active) * drun;
    grid = (int)(items < (long long)kCtasPerSm * sms ? items : (long long)kCtasPerSm * sms);
    if (grid > 0) {
        down_kernel<<<grid, kThreads, 0, st>>>(P);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace moe
