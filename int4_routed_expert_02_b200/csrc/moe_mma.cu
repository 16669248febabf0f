// moe_mma.cu -- tensor-core grouped GEMM for the expert FFN of a chunk of many
// tokens (prefill), on the 5th-generation tensor cores (tcgen05, TMEM).
//
// TurboFieldfare introduction page (discuss.pytorch.kr), section
// "TurboFieldfare's expert streaming structure": the prompt is prefilled in
// chunks of up to 128 tokens so that one read of an expert serves every row
// routed to it.  After bucketing, the rows of each expert form a small GEMM
//     g, u = Wg x, Wu x      (gate/up: [I, H] x [H, n])
//     a    = silu(g) * u
//     y    = Wd a            (down:    [H, I] x [I, n])
// with the weights in MLX affine 4-bit form (section "How TurboFieldfare saves
// memory": groups of 64 along the input, a BF16 scale and bias per group).
//
// One persistent CTA per SM walks a list of tiles.  A tile is 128 weight rows
// (the MMA's M) by the n <= 128 tokens of one expert (the MMA's N, padded to a
// multiple of 16), over the whole input dimension in k-blocks of 64 (one
// quantisation group, one 128-byte swizzle row of FP16):
//   weight producer  loads the tiled 4-bit codes and (scale, bias) words of
//                    the tile into a ring with 3-D TMA tensor copies (one box
//                    of 4 row blocks x a code stage per matrix);
//   token producer   loads the tokens' FP16 rows with 2-D TMA tensor copies
//                    (128-byte swizzle), in a warp of its own so that neither
//                    producer waits behind the other;
//   16 dequant warps turn each k-block of codes into FP16 weights
//                    w = s*q + b (exact q, one rounding) and store them into
//                    tensor memory (tcgen05.st: TMEM lane = tile row, two
//                    weights per 32-bit column), where the MMA reads its A
//                    operand -- so the FP16 weights never pass through shared
//                    memory, whose bandwidth an MMA with few tokens (small N)
//                    would otherwise spend mostly on re-reading A;
//   MMA thread       issues tcgen05.mma kind::f16 with A in TMEM and B (the
//                    tokens) in shared memory (FP16 x FP16 -> FP32 in TMEM)
//                    and signals buffers free with tcgen05.commit;
//   4 epilogue warps read the accumulators with tcgen05.ld (warp w: TMEM
//                    lanes 32 (w % 4) ..): gate/up tiles hold 128 gate rows in
//                    accumulator columns [0, N) and the same 128 up rows in
//                    [N, 2N), so each thread forms a = silu(g) * u for its row
//                    and writes it as FP16 -- the down GEMM's B operand; down
//                    tiles write fp32 y rows for the combine.  The accumulator
//                    is double-buffered (two 128-column buffers, tiles wider
//                    than 128 columns take both), so the MMAs of the next tile
//                    run while the epilogue drains this one, and the dequant
//                    warps never wait for an epilogue.
//
// Operand precision.  The tensor cores take FP16 or BF16 at the same rate and
// the same bytes.  FP16 is used: its 11-bit significand keeps the rounding of
// w = s*q + b and of the SwiGLU output 8x finer than BF16's 8 bits (BF16
// operands cost up to ~2e-2 * rms of the layer output, the whole error budget;
// FP16 ~1e-3).  The activations convert exactly (a BF16 value of the
// normalised input has 8 significant bits and |x| <= sqrt(H)).  FP16's range
// is the price: a weight s*q + b or a SwiGLU output beyond +-65504 cannot be
// represented.  The dequant warps test every group's extremes (q = 0 and
// q = 15) and the epilogue every SwiGLU value; the first value out of range
// is recorded in a status word of its own (range_err), which no wait polls,
// so the kernels run to their end and the call reports the layer as outside
// this path's domain instead of returning a silently saturated result.
//
// K order inside a chunk of 8.  The dequantisation makes BF16 pairs from
// nibbles j and j+4 of a word (one mask per pair), so the 8 weights of a
// 16-byte chunk are stored in the order (0,4,1,5,2,6,3,7) of their input
// index.  The activations are stored with the same order inside every chunk
// (by the gather kernel, and by the gate/up epilogue for the down GEMM), so the
// products pair up exactly and the dot product is unchanged.
//
// Every wait is bounded (~1 s of globaltimer); on a timeout the kernel records
// an error code, stops, waits (bounded) for its own copies and MMAs, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace mma {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 64;           // input columns per k-block
constexpr int kKS = 2;            // k-blocks per code stage
constexpr int kCodeSlots = 8;     // code stages in flight
constexpr int kABufs = 4;         // FP16 weight stages in TMEM (64 columns each)
constexpr int kBBufs = 3;         // token slots of 16 KiB: 128 / N k-blocks of an N-token tile each
constexpr int kMaxN = 128;        // tokens per tile
constexpr int kBoxRows = 16;      // rows of one TMA box of the token matrix
constexpr int kDqWarps = 16;      // dequant warps: one 32-code record per thread per stage
constexpr int kProdWarp = 16;   // weight codes
constexpr int kMmaWarp = 17;
constexpr int kTokWarp = 18;    // token tiles
constexpr int kEpiWarp0 = 19;   // 4 epilogue warps: warp w reads TMEM lanes 32 * (w % 4) ..
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kTmemCols = 512;   // accumulators in columns [0, 256), weight stages in [256, 512)
constexpr int kAccCols = 256;     // two accumulator buffers of 128 columns; a tile wider than 128 takes both
constexpr int kAStageCols = 64;   // 2 tiles of 128 x 64 FP16 (32 columns each)
constexpr int kBBufBytes = kMaxN * kBK * 2;      // 16 KiB
constexpr int kBoxBytes = kBoxRows * kBK * 2;    // 2 KiB
constexpr unsigned long long kWaitNs = 1000000000ull;

enum { kErrCodeFull = 1, kErrCodeEmpty, kErrAFull, kErrAEmpty, kErrBFull, kErrBEmpty, kErrAccFull, kErrAccEmpty };

// Shared-memory plan of the kernel for NMAT weight matrices per tile (2:
// gate and up, 1: down).  A weight stage (in TMEM) holds kAK k-blocks of
// every matrix (NMAT * kAK = 2 tiles of 128 x 64 FP16), so that each of the
// 512 dequant threads converts exactly one 32-code record per stage.
template <int NMAT>
struct Lay {
    static constexpr int kAK = 2 / NMAT;
    static constexpr int kCodeBytes = NMAT * 4 * kKS * 1024;
    static constexpr int kSbBytes = NMAT * 4 * kKS * 128;
    static constexpr int kSlotBytes = kCodeBytes + kSbBytes;
    static constexpr int kBOff = 0;
    static constexpr int kCodeOff = kBOff + kBBufs * kBBufBytes;
    static constexpr int kBarOff = kCodeOff + kCodeSlots * kSlotBytes;
    static constexpr int kNumBars = 2 * kCodeSlots + 2 * kABufs + 2 * kBBufs + 6;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kTmemSlotOff + 16;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 bytes
};
static_assert(Lay<2>::kAlloc <= 227 * 1024, "gate/up tile buffers exceed shared memory");
static_assert(kAccCols + kABufs * kAStageCols <= kTmemCols && 2 * kMaxN <= kAccCols, "tensor memory plan");
static_assert(kDqWarps * 32 == 2 * 2 * kBM, "one record (row, 32 codes) per dequant thread and stage");
static_assert(kKS % Lay<1>::kAK == 0 && kKS % Lay<2>::kAK == 0, "a code stage holds whole weight stages");

struct Params {
    const uint32_t *q[2], *sb[2];    // routed matrices (tiled layout), stacked over experts
    const uint32_t *sq[2], *ssb[2];  // the shared expert's
    int rows_r, rows_s;              // output rows of a routed / the shared matrix
    int K_r, K_s;                    // input columns of a routed / the shared matrix
    int T, k, with_shared, nt_max, n_items;
    const int32_t *offsets, *perm, *active;
    uint16_t *act;  // gate/up output [R, act_ld] FP16, chunk-permuted: shared rows [0,T), routed [T + pos]
    int act_ld;
    float *y;   // down output, routed: [T*k, H] by pair id
    float *sh;  // down output, shared: [T, H]
    int H;
    int *err;        // bounded-wait timeouts (every wait polls it and stops)
    int *range_err;  // a weight or SwiGLU value outside the FP16 range (no wait polls it)
    int test_stall;  // tests of the timeout path: the epilogue first waits on a barrier nothing arrives at
};

// TMA tensor maps of one launch: the token matrix (B operand) and the tiled
// codes / (scale, bias) words of the routed matrices (q, sb) and of the
// shared expert's (sq, ssb), each viewed as [row blocks][chunks or groups][32 lanes x words].
struct Maps {
    CUtensorMap tok;
    CUtensorMap q[2], sb[2], sq[2], ssb[2];
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t b, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t b, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t b, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(b), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with `parity` to complete; false on a timeout or
// when another thread has recorded an error.  sleep_ns > 0 backs off between
// tests: the producers, which run ahead, then leave the issue slots of their
// SM sub-partition to the dequantising warps that share it.
__device__ bool mbar_wait(uint32_t b, unsigned parity, int *err, int code, unsigned sleep_ns = 0) {
    if (mbar_test(b, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 1;; ++it) {
        if (sleep_ns) __nanosleep(sleep_ns);
        if (mbar_test(b, parity)) return true;
        if ((it & 63u) == 0) {
            if (__ldcg(err) != 0) return false;
            if (globaltimer() - t0 > kWaitNs) {
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// Bounded wait used when stopping: ignores the error flag.
__device__ void mbar_drain(uint32_t b, unsigned parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_test(b, parity)) {
        if (globaltimer() - t0 > kWaitNs) return;
    }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, unsigned bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// 3-D tiled TMA load (no multicast): box at (x, y, z) of the tensor map.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// 2-D tiled TMA load (no multicast): box at (x = column, y = row) of the tensor map.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle
// layout (8-row atoms of 1024 bytes, atoms stacked every 1024 bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)  // start address
           | ((uint64_t)1 << 16)                // leading byte offset (unused in this layout)
           | ((uint64_t)(1024 >> 4) << 32)      // stride byte offset: next 8-row atom
           | ((uint64_t)1 << 46)                // descriptor version
           | ((uint64_t)2 << 61);               // 128-byte swizzle
}

// Instruction descriptor, kind::f16: A and B FP16 (format 0, K-major), D FP32, M = 128.
__device__ __forceinline__ uint32_t idesc_f16(int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// The same with A read from tensor memory at a_tmem (lane 0 = row 0 of the
// 128-row operand, 16 K-elements in 8 consecutive 32-bit columns).
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, int acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// One thread's 16 consecutive 32-bit columns of its TMEM lane (a warp stores
// its 32 lanes; the address's lane field must be the warp's lane quarter).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint4 (&v)[4]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0].x), "r"(v[0].y), "r"(v[0].z), "r"(v[0].w), "r"(v[1].x), "r"(v[1].y), "r"(v[1].z), "r"(v[1].w),
        "r"(v[2].x), "r"(v[2].y), "r"(v[2].z), "r"(v[2].w), "r"(v[3].x), "r"(v[3].y), "r"(v[3].z), "r"(v[3].w)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Two fp32 values -> packed FP16 pair (lo, hi), round to nearest even.
__device__ __forceinline__ uint32_t f16x2_from_f32(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Packed BF16 pair -> packed FP16 pair (exact for the values of a normalised input).
__device__ __forceinline__ uint32_t f16x2_from_bf16x2(uint32_t v) {
    return f16x2_from_f32(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// 8 codes of one word -> 8 FP16 weights s*q + b, in the chunk order
// (0,4,1,5,2,6,3,7).  A code moved to mantissa bits 6..9 of an FP16 half with
// a zero exponent is the subnormal q * 2^-18, so one FMA with the scale
// pre-multiplied by 2^18 (s2) and the bias gives s*q + b with a single
// rounding.  Valid while s * 2^18 fits FP16 (|s| < 0.25).
__device__ __forceinline__ uint4 dequant_word_sub(uint32_t w, uint32_t s2, uint32_t b2) {
    constexpr uint32_t kM = 0x03C003C0u;
    return make_uint4(h2_fma((w << 6) & kM, s2, b2), h2_fma((w << 2) & kM, s2, b2), h2_fma((w >> 2) & kM, s2, b2),
                      h2_fma((w >> 6) & kM, s2, b2));
}

// The same for any scale: 0x6400 | q is the FP16 number 1024 + q, so
// subtracting 1024 gives q exactly before the FMA with the scale and bias.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t s2, uint32_t b2) {
    constexpr uint32_t kM = 0x000F000Fu, kMagic = 0x64006400u, kOne = 0x3C003C00u, kNeg1024 = 0xE400E400u;
    const uint32_t p0 = h2_fma((w & kM) | kMagic, kOne, kNeg1024);
    const uint32_t p1 = h2_fma(((w >> 4) & kM) | kMagic, kOne, kNeg1024);
    const uint32_t p2 = h2_fma(((w >> 8) & kM) | kMagic, kOne, kNeg1024);
    const uint32_t p3 = h2_fma(((w >> 12) & kM) | kMagic, kOne, kNeg1024);
    return make_uint4(h2_fma(p0, s2, b2), h2_fma(p1, s2, b2), h2_fma(p2, s2, b2), h2_fma(p3, s2, b2));
}

// Position, inside its chunk of 8, at which input index j is stored.
__device__ __forceinline__ int chunk_pos(int j) { return ((j & 3) << 1) | (j >> 2); }

// ------------------------------------------------------------------ tiles

struct Tile {
    int e;     // routed expert, or -1 for the shared expert
    int mt;    // 128-row block of the output rows
    int rv;    // valid rows in it (a multiple of 32)
    int brow;  // first row of its tokens in the token matrix
    int n;     // tokens
    int N;     // MMA N: n rounded up to 16
    int K;     // input columns
    int seg0;  // shared: first token; routed: first bucketed position
};

// Tile `it` of the list: the shared expert's tiles first (token blocks x row
// blocks), then each active expert's (token blocks x row blocks).  False for
// an empty slot of the list.
__device__ __forceinline__ bool get_tile(const Params &P, int it, Tile &t) {
    const int mt_s = (P.rows_s + kBM - 1) / kBM, mt_r = (P.rows_r + kBM - 1) / kBM;
    const int ns = P.with_shared ? mt_s * P.nt_max : 0;
    int rows, nt;
    if (it < ns) {
        nt = it / mt_s;
        t.mt = it - nt * mt_s;
        t.e = -1;
        t.seg0 = nt * kMaxN;
        t.n = min(kMaxN, P.T - t.seg0);
        t.brow = t.seg0;
        rows = P.rows_s;
        t.K = P.K_s;
    } else {
        const int per = P.nt_max * mt_r;
        const int j = it - ns;
        const int slot = j / per;
        const int r = j - slot * per;
        nt = r / mt_r;
        t.mt = r - nt * mt_r;
        if (slot >= __ldg(P.active)) return false;
        t.e = __ldg(P.active + 1 + slot);
        const int s0 = __ldg(P.offsets + t.e), cnt = __ldg(P.offsets + t.e + 1) - s0;
        if (nt * kMaxN >= cnt) return false;
        t.n = min(kMaxN, cnt - nt * kMaxN);
        t.seg0 = s0 + nt * kMaxN;
        t.brow = P.T + t.seg0;
        rows = P.rows_r;
        t.K = P.K_r;
    }
    if (t.n <= 0) return false;
    t.rv = min(kBM, rows - t.mt * kBM);
    t.N = (t.n + 15) & ~15;
    return true;
}

// ------------------------------------------------------------------ kernel

template <int NMAT>
__global__ void __launch_bounds__(kThreads, 1) expert_mma_kernel(const __grid_constant__ Params P,
                                                                 const __grid_constant__ Maps M) {
    const CUtensorMap &tmB = M.tok;
    using L = Lay<NMAT>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *gbase = smem_raw + (base - raw);
    const uint32_t sB = base + L::kBOff, sC = base + L::kCodeOff;
    const uint32_t bars = base + L::kBarOff;
    auto code_full = [&](int i) { return bars + 8u * i; };
    auto code_empty = [&](int i) { return bars + 8u * (kCodeSlots + i); };
    auto a_full = [&](int i) { return bars + 8u * (2 * kCodeSlots + i); };
    auto a_empty = [&](int i) { return bars + 8u * (2 * kCodeSlots + kABufs + i); };
    auto b_full = [&](int i) { return bars + 8u * (2 * kCodeSlots + 2 * kABufs + i); };
    auto b_empty = [&](int i) { return bars + 8u * (2 * kCodeSlots + 2 * kABufs + kBBufs + i); };
    // accumulator buffer i (columns [128 i, 128 i + 128)): full (MMAs done) and empty (epilogue done)
    auto acc_full = [&](int i) { return bars + 8u * (2 * kCodeSlots + 2 * kABufs + 2 * kBBufs + i); };
    auto acc_empty = [&](int i) { return bars + 8u * (2 * kCodeSlots + 2 * kABufs + 2 * kBBufs + 2 + i); };
    const uint32_t drain = bars + 8u * (2 * kCodeSlots + 2 * kABufs + 2 * kBBufs + 4);
    const uint32_t stall = bars + 8u * (2 * kCodeSlots + 2 * kABufs + 2 * kBBufs + 5);  // never arrived at
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::kTmemSlotOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kCodeSlots; ++i) {
            mbar_init(code_full(i), 1);
            mbar_init(code_empty(i), kDqWarps);
        }
        for (int i = 0; i < kABufs; ++i) {
            mbar_init(a_full(i), kDqWarps);
            mbar_init(a_empty(i), 1);
        }
        for (int i = 0; i < kBBufs; ++i) {
            mbar_init(b_full(i), 1);
            mbar_init(b_empty(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full(i), 1);
            mbar_init(acc_empty(i), kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(stall, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProdWarp) {
        // ---------------------------------------------------------- weight producer
        if (lane == 0) {
            uint32_t cs = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
                Tile t;
                if (!get_tile(P, it, t)) continue;
                const int nkb = t.K / kBK;
                const int mrb0 = (t.e < 0 ? 0 : t.e * (P.rows_r / 32)) + t.mt * 4;  // first row block of the tile
                for (int kb = 0; kb < nkb; kb += kKS) {
                    const int s = cs % kCodeSlots;
                    if (cs >= kCodeSlots &&
                        !mbar_wait(code_empty(s), ((cs / kCodeSlots) & 1) ^ 1, P.err, kErrCodeEmpty, 256)) {
                        ok = false;
                        break;
                    }
                    // whole boxes always land (out-of-range rows and chunks are zero-filled)
                    mbar_expect_tx(code_full(s), (unsigned)L::kSlotBytes);
                    const uint32_t slot = sC + (uint32_t)s * L::kSlotBytes;
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) {
                        tma_load_3d(slot + (uint32_t)(m * 4 * kKS) * 1024u, t.e < 0 ? &M.sq[m] : &M.q[m], 0, 2 * kb,
                                    mrb0, code_full(s));
                        tma_load_3d(slot + L::kCodeBytes + (uint32_t)(m * 4 * kKS) * 128u, t.e < 0 ? &M.ssb[m] : &M.sb[m],
                                    0, kb, mrb0, code_full(s));
                    }
                    ++cs;
                }
            }
            // let this lane's copies land before the CTA stops (bounded)
            for (uint32_t c = cs > (uint32_t)kCodeSlots ? cs - kCodeSlots : 0u; c < cs; ++c)
                mbar_drain(code_full(c % kCodeSlots), (c / kCodeSlots) & 1);
        }
    } else if (warp == kTokWarp) {
        // ---------------------------------------------------------- token producer
        if (lane == 0) {
            uint32_t kbc = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
                Tile t;
                if (!get_tile(P, it, t)) continue;
                const int nkb = t.K / kBK, nbox = t.N / kBoxRows, bkb = kMaxN / t.N;  // k-blocks per token slot
                for (int kb = 0; kb < nkb; kb += bkb) {
                    const int b = kbc % kBBufs;
                    if (kbc >= kBBufs && !mbar_wait(b_empty(b), ((kbc / kBBufs) & 1) ^ 1, P.err, kErrBEmpty, 256)) {
                        ok = false;
                        break;
                    }
                    const int nk = min(bkb, nkb - kb);
                    mbar_expect_tx(b_full(b), (unsigned)(nk * nbox * kBoxBytes));
                    for (int i = 0; i < nk; ++i)
                        for (int j = 0; j < nbox; ++j)
                            tma_load_2d(sB + (uint32_t)b * kBBufBytes + (uint32_t)((i * nbox + j) * kBoxBytes), &tmB,
                                        (kb + i) * kBK, t.brow + j * kBoxRows, b_full(b));
                    ++kbc;
                }
            }
            for (uint32_t c = kbc > (uint32_t)kBBufs ? kbc - kBBufs : 0u; c < kbc; ++c)
                mbar_drain(b_full(c % kBBufs), (c / kBBufs) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t asc = 0, kbc = 0, ic = 0;
            bool ok = true, prev_wide = false;
            for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
                Tile t;
                if (!get_tile(P, it, t)) continue;
                // tile ic accumulates in buffer ic % 2, or in both when wider than one;
                // wait until the epilogue has drained the last tile whose columns it
                // overwrites (tiles are drained in order, so tile j's count implies
                // every earlier one's)
                const bool wide = NMAT * t.N > kAccCols / 2;
                const int need = (wide || prev_wide) ? (int)ic - 1 : (int)ic - 2;
                prev_wide = wide;
                if (need >= 0) {
                    if (!mbar_wait(acc_empty(need & 1), (need >> 1) & 1, P.err, kErrAccEmpty)) break;
                    tc_fence_after();
                }
                const uint32_t dacc = tmem + (wide ? 0u : (ic & 1u) * (uint32_t)(kAccCols / 2));
                const uint32_t idesc = idesc_f16(t.N);
                const int nkb = t.K / kBK, bkb = kMaxN / t.N;
                const uint32_t bstep = (uint32_t)t.N * kBK * 2;  // bytes of one k-block of the tile's tokens
                int kin = 0;                                      // k-block inside the current token slot
                // one issuing thread: keep the per-MMA work to adds (descriptors and
                // addresses advance by constants, no division in the loop)
                for (int ks = 0; ks < nkb && ok; ks += L::kAK) {
                    const int a = asc % kABufs;
                    if (!mbar_wait(a_full(a), (asc / kABufs) & 1, P.err, kErrAFull)) {
                        ok = false;
                        break;
                    }
                    const uint32_t abase = tmem + (uint32_t)(kAccCols + a * kAStageCols);
                    for (int kbi = 0; kbi < L::kAK && ks + kbi < nkb; ++kbi) {
                        const int kb = ks + kbi, b = kbc % kBBufs;
                        if (kin == 0 && !mbar_wait(b_full(b), (kbc / kBBufs) & 1, P.err, kErrBFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t bdesc = sw128_desc(sB + (uint32_t)b * kBBufBytes + (uint32_t)kin * bstep);
                        const uint32_t a0 = abase + (uint32_t)(kbi * 32);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                            for (int m = 0; m < NMAT; ++m)  // +32 bytes of K: +2 in the descriptor's address field
                                mma_f16_tmem_a(dacc + (uint32_t)(m * t.N), a0 + (uint32_t)(m * L::kAK * 32 + kk * 8),
                                               bdesc + (uint64_t)(2 * kk), idesc, (kb | kk) != 0);
                        }
                        if (++kin == bkb || kb == nkb - 1) {  // last k-block of this token slot
                            mma_commit(b_empty(b));
                            ++kbc;
                            kin = 0;
                        }
                    }
                    if (!ok) break;
                    mma_commit(a_empty(a));
                    ++asc;
                }
                if (!ok) break;
                mma_commit(acc_full(ic & 1));
                ++ic;
            }
            // every MMA this thread issued has completed once `drain` fires
            mma_commit(drain);
            mbar_drain(drain, 0);
        }
    } else if (warp < kDqWarps) {
        // ---------------------------------------------------------- dequant
        // thread -> one record per weight stage: tile row r, matrix m, k-block kbi of the stage, 32-code half
        const int r = threadIdx.x & (kBM - 1), j4 = threadIdx.x >> 7;
        const int m = NMAT == 2 ? (j4 >> 1) : 0, kbi = NMAT == 2 ? 0 : (j4 >> 1), half = j4 & 1;
        const int rbl = r >> 5, rl = r & 31;
        uint32_t cs = 0, asc = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
            Tile t;
            if (!get_tile(P, it, t)) continue;
            const int nkb = t.K / kBK;
            for (int ks = 0; ks < nkb; ks += L::kAK) {
                const int s = cs % kCodeSlots, kbs = ks % kKS + kbi;
                if (ks % kKS == 0 && !__all_sync(0xffffffffu, mbar_wait(code_full(s), (cs / kCodeSlots) & 1, P.err,
                                                                          kErrCodeFull))) {
                    ok = false;
                    break;
                }
                const unsigned char *slot = gbase + L::kCodeOff + (size_t)s * L::kSlotBytes;
                const bool valid = r < t.rv && ks + kbi < nkb;
                uint4 c = make_uint4(0u, 0u, 0u, 0u);
                uint32_t sbw = 0;
                if (valid) {
                    c = *reinterpret_cast<const uint4 *>(slot + ((((m * 4 + rbl) * kKS + kbs) * 2 + half) * 512) + rl * 16);
                    sbw = *reinterpret_cast<const uint32_t *>(slot + L::kCodeBytes + (((m * 4 + rbl) * kKS + kbs) * 32 + rl) * 4);
                }
                if ((ks + L::kAK) % kKS == 0 || ks + L::kAK >= nkb) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(code_empty(s));
                    ++cs;
                }
                const int a = asc % kABufs;
                if (asc >= kABufs &&
                    !__all_sync(0xffffffffu, mbar_wait(a_empty(a), ((asc / kABufs) & 1) ^ 1, P.err, kErrAEmpty))) {
                    ok = false;
                    break;
                }
                tc_fence_after();  // the MMAs that read this stage's columns have completed
                if (valid) {  // warp-uniform: rv is a multiple of 32, kbi is the warp's
                    const float sf = __uint_as_float(sbw << 16), bf = __uint_as_float(sbw & 0xffff0000u);
                    // s*q + b is linear in q: its extremes over the group are at q = 0 and q = 15
                    if (!(fmaxf(fabsf(bf), fabsf(fmaf(15.0f, sf, bf))) <= 65504.0f)) atomicCAS(P.range_err, 0, 1);
                    const uint32_t b2 = f16x2_from_f32(bf, bf);
                    const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
                    uint4 o[4];
                    if (fabsf(sf) < 0.25f) {
                        const uint32_t s2 = f16x2_from_f32(sf * 262144.0f, sf * 262144.0f);
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) o[wi] = dequant_word_sub(wv[wi], s2, b2);
                    } else {
                        const uint32_t s2 = f16x2_from_f32(sf, sf);
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) o[wi] = dequant_word(wv[wi], s2, b2);
                    }
                    // columns: stage a, tile (m, kbi), this half's 16 columns; lane field: this warp's rows
                    tmem_st16(tmem + ((uint32_t)(r & ~31) << 16) +
                                  (uint32_t)(kAccCols + a * kAStageCols + (m * L::kAK + kbi) * 32 + half * 16),
                              o);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(a_full(a));
                ++asc;
            }
        }
    } else if (warp >= kEpiWarp0) {
        // ---------------------------------------------------------- epilogue
        // warp w reads TMEM lanes 32*(w%4).. (tile rows); tiles in order, buffers alternating
        const int q4 = warp & 3;
        uint32_t ic = 0;
        // test hook: a wait that runs out (about 1 s); every role then stops as on a real timeout
        const bool stalled =
            P.test_stall && !__all_sync(0xffffffffu, mbar_wait(stall, 0, P.err, kErrAccFull));
        for (int it = stalled ? P.n_items : (int)blockIdx.x; it < P.n_items; it += gridDim.x) {
            Tile t;
            if (!get_tile(P, it, t)) continue;
            const int ab = (int)(ic & 1u);
            if (!__all_sync(0xffffffffu, mbar_wait(acc_full(ab), (ic >> 1) & 1, P.err, kErrAccFull))) break;
            tc_fence_after();
            const bool wide = NMAT * t.N > kAccCols / 2;
            const int row = t.mt * kBM + q4 * 32 + lane;
            const bool rvalid = q4 * 32 < t.rv;  // warp-uniform
            const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) + (wide ? 0u : (uint32_t)ab * (kAccCols / 2));
            if (rvalid) {
                for (int ch = 0; ch < t.N / 8; ++ch) {
                    if (NMAT == 2) {
                        float g[8], u[8];
                        tmem_ld8(taddr + ch * 8, g);
                        tmem_ld8(taddr + t.N + ch * 8, u);
                        const int col = (row & ~7) | chunk_pos(row & 7);
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int n = ch * 8 + jj;
                            if (n < t.n) {
                                float av = silu_mul(g[jj], u[jj]);
                                if (!(fabsf(av) <= 65504.f)) {
                                    atomicCAS(P.range_err, 0, 2);
                                    av = 0.f;  // the call is reported as outside this path's domain
                                }
                                P.act[(size_t)(t.brow + n) * P.act_ld + col] = __half_as_ushort(__float2half_rn(av));
                            }
                        }
                    } else {
                        float v[8];
                        tmem_ld8(taddr + ch * 8, v);
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int n = ch * 8 + jj;
                            if (n < t.n) {
                                if (t.e < 0)
                                    P.sh[(size_t)(t.seg0 + n) * P.H + row] = v[jj];
                                else
                                    P.y[(size_t)__ldg(P.perm + t.seg0 + n) * P.H + row] = v[jj];
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(ab));
            ++ic;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// Token matrix for the gate/up GEMM, FP16: row r < T is token r, row T + j the
// token of bucketed pair j; every 16-byte chunk stored in the order
// (0,4,1,5,2,6,3,7).  The pairs (1,5) and (3,7) are multiplied by odd_scale
// (1, or 1/16 for the warp-MMA path) before their one rounding to FP16.
__global__ void __launch_bounds__(256) gather_kernel(const uint16_t *__restrict__ xe, const int32_t *__restrict__ perm,
                                                     int T, int k, int H, int R, float odd_scale,
                                                     uint16_t *__restrict__ xg) {
    const int cpr = H / 8;  // 16-byte chunks per row
    const long long total = (long long)R * cpr;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i / cpr), c = (int)(i - (long long)r * cpr);
        const int tok = r < T ? r : __ldg(perm + (r - T)) / k;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xe + (size_t)tok * H) + c);
        uint4 o;  // pairs (0,4), (1,5), (2,6), (3,7), each converted BF16 -> FP16
        o.x = f16x2_from_bf16x2(__byte_perm(v.x, v.z, 0x5410));
        const uint32_t p15 = __byte_perm(v.x, v.z, 0x7632), p37 = __byte_perm(v.y, v.w, 0x7632);
        o.y = f16x2_from_f32(__uint_as_float(p15 << 16) * odd_scale, __uint_as_float(p15 & 0xffff0000u) * odd_scale);
        o.z = f16x2_from_bf16x2(__byte_perm(v.y, v.w, 0x5410));
        o.w = f16x2_from_f32(__uint_as_float(p37 << 16) * odd_scale, __uint_as_float(p37 & 0xffff0000u) * odd_scale);
        reinterpret_cast<uint4 *>(xg + (size_t)r * H)[c] = o;
    }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Row-major FP16 matrix [rows, cols] (row stride ld elements), boxes of 16 rows x 64 columns, 128-byte swizzle.
static cudaError_t make_map(CUtensorMap *m, const uint16_t *ptr, int rows, int cols, int ld) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBoxRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Tiled codes [n_rb][C][128 u32] or (scale, bias) words [n_rb][G][32 u32] of a
// matrix set, boxes of 4 row blocks x `per` chunks (or groups) x all lanes.
static cudaError_t make_qmap(CUtensorMap *m, const uint32_t *ptr, int n_rb, int per_rb, int words, int per) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)words, (cuuint64_t)per_rb, (cuuint64_t)n_rb};
    const cuuint64_t strides[2] = {(cuuint64_t)words * 4, (cuuint64_t)words * 4 * per_rb};
    const cuuint32_t box[3] = {(cuuint32_t)words, (cuuint32_t)per, 4};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Maps of the routed matrices q/sb[0..nmat) ([n_mat][rows][K] each) and of the shared ones ([rows_s][K_s]).
static cudaError_t make_weight_maps(Maps &M, const Params &P, int nmat, int n_mat) {
    for (int m = 0; m < nmat; ++m) {
        cudaError_t e = make_qmap(&M.q[m], P.q[m], n_mat * P.rows_r / 32, P.K_r / 32, 128, 2 * kKS);
        if (e == cudaSuccess) e = make_qmap(&M.sb[m], P.sb[m], n_mat * P.rows_r / 32, P.K_r / 64, 32, kKS);
        if (e == cudaSuccess && P.with_shared) e = make_qmap(&M.sq[m], P.sq[m], P.rows_s / 32, P.K_s / 32, 128, 2 * kKS);
        if (e == cudaSuccess && P.with_shared) e = make_qmap(&M.ssb[m], P.ssb[m], P.rows_s / 32, P.K_s / 64, 32, kKS);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <int NMAT>
static cudaError_t launch_mma(Params &P, const Maps &map, int max_items, cudaStream_t st) {
    using Lt = Lay<NMAT>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(expert_mma_kernel<NMAT>), Lt::kAlloc);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorNoDevice;
    P.n_items = max_items;
    const int grid = max_items < sms ? max_items : sms;
    if (grid <= 0) return cudaSuccess;
    expert_mma_kernel<NMAT><<<grid, kThreads, Lt::kAlloc, st>>>(P, map);
    return cudaGetLastError();
}

}  // namespace mma

cudaError_t launch_gather_tokens(const uint16_t *xe, const int32_t *perm, int T, int k, int H, uint16_t *xg,
                                 cudaStream_t st, bool odd_div16) {
    const int R = T + T * k;
    const long long chunks = (long long)R * (H / 8);
    long long blocks = (chunks + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    if (blocks <= 0) return cudaSuccess;
    mma::gather_kernel<<<(int)blocks, 256, 0, st>>>(xe, perm, T, k, H, R, odd_div16 ? 0.0625f : 1.0f, xg);
    return cudaGetLastError();
}

size_t mma_xg_bytes(const moe_layer_w *w, int T) {
    return sizeof(uint16_t) * ((size_t)T + (size_t)T * w->k) * w->H;
}
size_t mma_act_bytes(const moe_layer_w *w, int T) {
    const int Kmax = w->I > w->Is ? w->I : w->Is;
    return sizeof(uint16_t) * ((size_t)T + (size_t)T * w->k) * Kmax;
}

cudaError_t launch_expert_mma(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                              const int32_t *perm, const int32_t *active, int with_shared, const MmaBuffers &b,
                              cudaStream_t st) {
    using namespace mma;
    const int H = w->H, k = w->k, I = w->I, Is = w->Is;
    const int Kmax = I > Is ? I : Is;
    const int R = T + T * k;
    {
        cudaError_t e = launch_gather_tokens(xe, perm, T, k, H, b.xg, st);
        if (e != cudaSuccess) return e;
    }
    static thread_local Maps mx, ma;  // large; kept off the stack
    cudaError_t e = make_map(&mx.tok, b.xg, R, H, H);
    if (e != cudaSuccess) return e;
    e = make_map(&ma.tok, b.act, R, Kmax, Kmax);
    if (e != cudaSuccess) return e;

    Params P{};
    P.T = T;
    P.k = k;
    P.with_shared = with_shared;
    P.nt_max = (T + kMaxN - 1) / kMaxN;
    P.offsets = offsets;
    P.perm = perm;
    P.active = active;
    P.act = b.act;
    P.act_ld = Kmax;
    P.y = b.y;
    P.sh = b.sh;
    P.H = H;
    P.err = b.err;
    P.range_err = b.range_err;
    // test hook: MOE_TEST_MMA_STALL=1 makes the epilogue's first wait run out, so that the
    // kernels' bounded waits and their report through the workspace status are exercised
    const char *stall_env = getenv("MOE_TEST_MMA_STALL");
    P.test_stall = (stall_env && stall_env[0] == '1') ? 1 : 0;
    const long long pairs = (long long)T * k;
    const int max_active = (int)(pairs < w->E ? pairs : w->E);

    // gate/up: rows I (Is) of two matrices, input H
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
    P.K_r = H;
    P.K_s = H;
    {
        const int mt_s = (Is + kBM - 1) / kBM, mt_r = (I + kBM - 1) / kBM;
        const int items = (with_shared ? mt_s * P.nt_max : 0) + max_active * P.nt_max * mt_r;
        e = make_weight_maps(mx, P, 2, w->E);
        if (e != cudaSuccess) return e;
        e = launch_mma<2>(P, mx, items, st);
        if (e != cudaSuccess) return e;
    }
    // down: rows H of one matrix, input I (Is)
    P.q[0] = w->down.q;
    P.sb[0] = w->down.sb;
    P.q[1] = nullptr;
    P.sb[1] = nullptr;
    P.sq[0] = w->sh_down.q;
    P.ssb[0] = w->sh_down.sb;
    P.sq[1] = nullptr;
    P.ssb[1] = nullptr;
    P.rows_r = H;
    P.rows_s = H;
    P.K_r = I;
    P.K_s = Is;
    {
        const int mt = (H + kBM - 1) / kBM;
        const int items = (with_shared ? mt * P.nt_max : 0) + max_active * P.nt_max * mt;
        e = make_weight_maps(ma, P, 1, w->E);
        if (e != cudaSuccess) return e;
        e = launch_mma<1>(P, ma, items, st);
    }
    return e;
}

}  // namespace moe
