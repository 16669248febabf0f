// moe_gemv.cu -- int4 dequant-GEMV for the routed and shared experts.
//
// Expert FFN (TurboFieldfare introduction page, discuss.pytorch.kr, section
// "TurboFieldfare's expert streaming structure": 8 routed experts per token
// out of 128, plus a shared branch without routing weight; weights are MLX
// affine 4-bit in groups of 64 with a BF16 scale and bias, section "How
// TurboFieldfare saves memory"):
//     g = Wg x,  u = Wu x,  a = silu(g) * u,  y = Wd a,   W = scale * q + bias.
//
// Design (B200, HBM-bound at decode batch sizes):
//  * Weights are in the tiled layout of moe_qmat: a warp's 32 lanes are 32
//    consecutive rows, and each 16-byte load of a lane is 32 codes of its
//    row, so one warp load instruction moves 512 contiguous bytes.  Each lane
//    accumulates its own row: no cross-lane reduction in the inner loop.
//  * One CTA = one 32-row block of one matrix (gate+up fused, or down) for
//    the tokens of one expert segment; its warps split the input dimension by
//    whole groups and are reduced through shared memory in a fixed order.
//  * The input vector is broadcast from shared memory, pre-scaled so that a
//    single FMA per code accumulates q*x exactly (see decode_word); the affine
//    part is applied per group as  s * sum(q x) + b * sum(x).
//  * The shared expert's row blocks come first in the grid; routed blocks for
//    slots beyond the number of experts actually used exit at once.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// ------------------------------------------------------------ repacking

__global__ void prepare_q_kernel(const uint32_t *__restrict__ q, int n_mat, int rows, int cols,
                                 uint32_t *__restrict__ q_out) {
    const int C = cols / kChunkCols, RB = rows / kRowBlock;
    const size_t units = (size_t)n_mat * RB * C * kWarp;  // one 16-byte unit each
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units; u += (size_t)gridDim.x * blockDim.x) {
        const int lane = (int)(u % kWarp);
        size_t r = u / kWarp;
        const int c = (int)(r % C);
        r /= C;
        const int rb = (int)(r % RB);
        const int m = (int)(r / RB);
        const size_t row = (size_t)m * rows + (size_t)rb * kRowBlock + lane;
        const uint4 v = *reinterpret_cast<const uint4 *>(q + row * (cols / 8) + 4 * (size_t)c);
        *reinterpret_cast<uint4 *>(q_out + 4 * u) = v;
    }
}

__global__ void prepare_sb_kernel(const uint16_t *__restrict__ s, const uint16_t *__restrict__ b, int n_mat,
                                  int rows, int cols, uint32_t *__restrict__ sb_out) {
    const int G = cols / kGroup, RB = rows / kRowBlock;
    const size_t units = (size_t)n_mat * RB * G * kWarp;
    for (size_t u = blockIdx.x * (size_t)blockDim.x + threadIdx.x; u < units; u += (size_t)gridDim.x * blockDim.x) {
        const int lane = (int)(u % kWarp);
        size_t r = u / kWarp;
        const int g = (int)(r % G);
        r /= G;
        const int rb = (int)(r % RB);
        const int m = (int)(r / RB);
        const size_t gi = ((size_t)m * rows + (size_t)rb * kRowBlock + lane) * G + g;
        sb_out[u] = (uint32_t)s[gi] | ((uint32_t)b[gi] << 16);
    }
}

cudaError_t launch_prepare_qmat(const uint32_t *q, const uint16_t *s, const uint16_t *b, int n_mat, int rows,
                                int cols, uint32_t *q_out, uint32_t *sb_out, cudaStream_t st) {
    prepare_q_kernel<<<1184, 256, 0, st>>>(q, n_mat, rows, cols, q_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prepare_sb_kernel<<<1184, 256, 0, st>>>(s, b, n_mat, rows, cols, sb_out);
    return cudaGetLastError();
}

// ------------------------------------------------------------ GEMV core

// Shared-memory staging of the inputs of one pass of up to NT tokens:
//   xp[NT][cols]      pre-scaled inputs x' = x * code_prescale(col % 8)
//   Xs[NT][cols/32]   sum of x over each 32-column chunk (for the bias term)
struct Stage {
    float *xp, *Xs;
    int cols, nchunk;
};

template <int NT>
__device__ __forceinline__ void stage_chunk_sums(const Stage &S, int nw) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float inv_scale = 1.0f / code_prescale(lane & 7);  // exact: a power of two
    for (int i = w; i < NT * S.nchunk; i += nw) {
        const int tt = i / S.nchunk, c = i - tt * S.nchunk;
        const float v = S.xp[(size_t)tt * S.cols + c * kChunkCols + lane];
        const float sx = warp_sum(v * inv_scale);
        if (lane == 0) S.Xs[i] = sx;
    }
}

// Accumulate, for NMAT matrices whose 32-row block starts at q[m] / sb[m],
// the dot products of this lane's row with the staged inputs over the groups
// [g0, g1).  acc[m][tt] receives  sum_groups  s * sum(q x) + b * sum(x).
template <int NT, int NMAT>
__device__ __forceinline__ void gemv_slice(const uint32_t *const (&q)[NMAT], const uint32_t *const (&sb)[NMAT],
                                           const Stage &S, int nt, int g0, int g1, float (&acc)[NMAT][NT]) {
    const int lane = threadIdx.x & 31;
    uint4 cur[NMAT][2], nxt[NMAT][2];
    uint32_t csb[NMAT], nsb[NMAT];
    if (g0 < g1) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            cur[m][0] = ldg_nc_v4(q[m] + (size_t)(2 * g0) * 128 + lane * 4);
            cur[m][1] = ldg_nc_v4(q[m] + (size_t)(2 * g0 + 1) * 128 + lane * 4);
            csb[m] = ldg_nc_u32(sb[m] + (size_t)g0 * 32 + lane);
        }
    }
    for (int g = g0; g < g1; ++g) {
        if (g + 1 < g1) {  // prefetch the next group while this one is computed
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                nxt[m][0] = ldg_nc_v4(q[m] + (size_t)(2 * g + 2) * 128 + lane * 4);
                nxt[m][1] = ldg_nc_v4(q[m] + (size_t)(2 * g + 3) * 128 + lane * 4);
                nsb[m] = ldg_nc_u32(sb[m] + (size_t)(g + 1) * 32 + lane);
            }
        }
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const float s = bf16_bits_to_float(csb[m] & 0xffffu) * kCodeUnscale;
            const float b = bf16_bits_to_float(csb[m] >> 16);
            const uint32_t words[8] = {cur[m][0].x, cur[m][0].y, cur[m][0].z, cur[m][0].w,
                                       cur[m][1].x, cur[m][1].y, cur[m][1].z, cur[m][1].w};
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                if (tt < nt) {
                    const float *xp = S.xp + (size_t)tt * S.cols + g * kGroup;
                    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int wi = 0; wi < 8; ++wi) dot_word(words[wi], xp + wi * 8, a0, a1);
                    const int ci = tt * S.nchunk + 2 * g;
                    acc[m][tt] = fmaf(s, (a0.x + a0.y) + (a1.x + a1.y), fmaf(b, S.Xs[ci] + S.Xs[ci + 1], acc[m][tt]));
                }
            }
        }
        if (g + 1 < g1) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                cur[m][0] = nxt[m][0];
                cur[m][1] = nxt[m][1];
                csb[m] = nsb[m];
            }
        }
    }
}

struct ExpertParams {
    // routed experts (tiled): gate/up E x [I, H], down E x [H, I]
    const uint32_t *gq, *gsb, *uq, *usb, *dq, *dsb;
    // shared expert (tiled): gate/up [Is, H], down [H, Is]
    const uint32_t *sgq, *sgsb, *suq, *susb, *sdq, *sdsb;
    const uint16_t *xe;  // [T, H] bf16
    const int32_t *offsets, *perm, *active;
    float *a_routed, *a_shared, *y, *sh;
    int T, H, I, Is, k, with_shared;
};

// Which work a CTA owns: a row block `rb` of the shared expert (`shared`), or
// of the routed expert in active slot `slot`, for n tokens starting at
// bucketed position seg0.  Returns false when the slot is unused.
struct Unit {
    bool shared;
    int rb, e, seg0, n;
};

__device__ __forceinline__ bool decode_unit(const ExpertParams &P, int rb_per_mat_shared, int rb_per_mat, Unit &u) {
    int b = blockIdx.x;
    const int nsh = P.with_shared ? rb_per_mat_shared : 0;
    if (b < nsh) {
        u.shared = true;
        u.rb = b;
        u.e = 0;
        u.seg0 = 0;
        u.n = P.T;
        return true;
    }
    b -= nsh;
    const int slot = b / rb_per_mat;
    u.shared = false;
    u.rb = b - slot * rb_per_mat;
    if (slot >= P.active[0]) return false;
    u.e = P.active[1 + slot];
    u.seg0 = P.offsets[u.e];
    u.n = P.offsets[u.e + 1] - u.seg0;
    return true;
}

// Token id of the j-th row of a unit.
__device__ __forceinline__ int unit_token(const ExpertParams &P, const Unit &u, int j) {
    return u.shared ? j : P.perm[u.seg0 + j] / P.k;
}

template <int NT, int NW>
__global__ void __launch_bounds__(NW * 32)
gateup_kernel(const ExpertParams P) {
    extern __shared__ __align__(16) float smem_f[];
    Unit u;
    if (!decode_unit(P, P.Is / kRowBlock, P.I / kRowBlock, u)) return;
    const int H = P.H, C = H / kChunkCols, G = H / kGroup;
    Stage S{smem_f, smem_f + (size_t)NT * H, H, C};
    float *red = S.Xs + NT * C;  // [2][NW][NT][32]
    const int rows = u.shared ? P.Is : P.I;
    const size_t mrb = u.shared ? (size_t)u.rb : (size_t)u.e * (rows / kRowBlock) + u.rb;
    const uint32_t *q[2] = {(u.shared ? P.sgq : P.gq) + mrb * C * 128, (u.shared ? P.suq : P.uq) + mrb * C * 128};
    const uint32_t *sb[2] = {(u.shared ? P.sgsb : P.gsb) + mrb * G * 32, (u.shared ? P.susb : P.usb) + mrb * G * 32};
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g0 = G * w / NW, g1 = G * (w + 1) / NW;

    for (int j0 = 0; j0 < u.n; j0 += NT) {
        const int nt = min(NT, u.n - j0);
        __syncthreads();
        for (int i = threadIdx.x; i < NT * H; i += blockDim.x) {
            const int tt = i / H, col = i - tt * H;
            float x = 0.f;
            if (tt < nt) x = bf16_bits_to_float(P.xe[(size_t)unit_token(P, u, j0 + tt) * H + col]);
            S.xp[i] = x * code_prescale(col & 7);
        }
        __syncthreads();
        stage_chunk_sums<NT>(S, NW);
        __syncthreads();
        float acc[2][NT];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) acc[m][tt] = 0.f;
        gemv_slice<NT, 2>(q, sb, S, nt, g0, g1, acc);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) red[((m * NW + w) * NT + tt) * 32 + lane] = acc[m][tt];
        __syncthreads();
        if (threadIdx.x < NT * 32) {
            const int tt = threadIdx.x >> 5;
            float gs = 0.f, us = 0.f;
            for (int ww = 0; ww < NW; ++ww) {  // fixed order: deterministic
                gs += red[((0 * NW + ww) * NT + tt) * 32 + lane];
                us += red[((1 * NW + ww) * NT + tt) * 32 + lane];
            }
            if (tt < nt) {
                const int row = u.rb * kRowBlock + lane;
                const float a = silu_mul(gs, us);
                if (u.shared)
                    P.a_shared[(size_t)(j0 + tt) * P.Is + row] = a;
                else
                    P.a_routed[(size_t)(u.seg0 + j0 + tt) * P.I + row] = a;
            }
        }
    }
}

template <int NT, int NW>
__global__ void __launch_bounds__(NW * 32)
down_kernel(const ExpertParams P) {
    extern __shared__ __align__(16) float smem_f[];
    Unit u;
    if (!decode_unit(P, P.H / kRowBlock, P.H / kRowBlock, u)) return;
    const int K = u.shared ? P.Is : P.I;  // input dimension of this matrix
    const int C = K / kChunkCols, G = K / kGroup;
    Stage S{smem_f, smem_f + (size_t)NT * K, K, C};
    float *red = S.Xs + NT * C;  // [NW][NT][32]
    const size_t mrb = u.shared ? (size_t)u.rb : (size_t)u.e * (P.H / kRowBlock) + u.rb;
    const uint32_t *q[1] = {(u.shared ? P.sdq : P.dq) + mrb * C * 128};
    const uint32_t *sb[1] = {(u.shared ? P.sdsb : P.dsb) + mrb * G * 32};
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g0 = G * w / NW, g1 = G * (w + 1) / NW;

    for (int j0 = 0; j0 < u.n; j0 += NT) {
        const int nt = min(NT, u.n - j0);
        __syncthreads();
        for (int i = threadIdx.x; i < NT * K; i += blockDim.x) {
            const int tt = i / K, col = i - tt * K;
            float x = 0.f;
            if (tt < nt) {
                x = u.shared ? P.a_shared[(size_t)(j0 + tt) * P.Is + col]
                             : P.a_routed[(size_t)(u.seg0 + j0 + tt) * P.I + col];
            }
            S.xp[i] = x * code_prescale(col & 7);
        }
        __syncthreads();
        stage_chunk_sums<NT>(S, NW);
        __syncthreads();
        float acc[1][NT];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) acc[0][tt] = 0.f;
        gemv_slice<NT, 1>(q, sb, S, nt, g0, g1, acc);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) red[(w * NT + tt) * 32 + lane] = acc[0][tt];
        __syncthreads();
        if (threadIdx.x < NT * 32) {
            const int tt = threadIdx.x >> 5;
            float ys = 0.f;
            for (int ww = 0; ww < NW; ++ww) ys += red[(ww * NT + tt) * 32 + lane];
            if (tt < nt) {
                const int row = u.rb * kRowBlock + lane;
                if (u.shared)
                    P.sh[(size_t)(j0 + tt) * P.H + row] = ys;
                else
                    P.y[(size_t)P.perm[u.seg0 + j0 + tt] * P.H + row] = ys;
            }
        }
    }
}

constexpr int kGateUpWarps = 8;
constexpr int kDownWarps = 4;

static size_t stage_bytes(int cols, int nt, int nred) {
    return sizeof(float) * ((size_t)nt * cols + (size_t)nt * (cols / kChunkCols) + (size_t)nred * nt * 32);
}

size_t gemv_smem_bytes(int cols, int nt) { return stage_bytes(cols, nt, 2 * kGateUpWarps); }

template <int NT>
static cudaError_t launch_ffn_nt(const ExpertParams &P, int max_active, cudaStream_t st) {
    const size_t s1 = stage_bytes(P.H, NT, 2 * kGateUpWarps);
    const size_t s2 = stage_bytes(P.Is > P.I ? P.Is : P.I, NT, kDownWarps);
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(gateup_kernel<NT, kGateUpWarps>), s1);
    if (e != cudaSuccess) return e;
    e = ensure_smem(reinterpret_cast<const void *>(down_kernel<NT, kDownWarps>), s2);
    if (e != cudaSuccess) return e;
    const int sh = P.with_shared ? 1 : 0;
    const int grid1 = sh * (P.Is / kRowBlock) + max_active * (P.I / kRowBlock);
    const int grid2 = sh * (P.H / kRowBlock) + max_active * (P.H / kRowBlock);
    if (grid1 > 0) gateup_kernel<NT, kGateUpWarps><<<grid1, kGateUpWarps * 32, s1, st>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (grid2 > 0) down_kernel<NT, kDownWarps><<<grid2, kDownWarps * 32, s2, st>>>(P);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ one large matrix
// y[t][r] = sum_c W[r][c] x[t][c] for a single tiled 4-bit matrix W [rows,
// cols], e.g. the vocabulary-sized output head that shares the embedding's
// quantised weights (TurboFieldfare introduction page, section "How
// TurboFieldfare saves memory": the embedding and the language-model head
// share the same quantised weights; the decode-time table there puts that
// head at 14.2 ms of a 162.8 ms step).  Pure streaming: every byte of W is
// read once, so the kernel is HBM-bound.  Each CTA stages x once; its warps
// then take 32-row blocks one at a time from a global counter (all rows of a
// block, every column), so no warp idles while another still streams.
constexpr int kQgWarps = 8;

template <int NT>
__global__ void __launch_bounds__(kQgWarps * 32)
qmat_gemv_kernel(const uint32_t *__restrict__ q, const uint32_t *__restrict__ sb, int rows, int cols,
                 const uint16_t *__restrict__ x, int T, float *__restrict__ y, unsigned *__restrict__ ctr) {
    extern __shared__ __align__(16) float smem_f[];
    const int C = cols / kChunkCols, G = cols / kGroup, nrb = rows / kRowBlock;
    Stage S{smem_f, smem_f + (size_t)NT * cols, cols, C};
    for (int i = threadIdx.x; i < NT * cols; i += blockDim.x) {
        const int tt = i / cols, col = i - tt * cols;
        const float v = tt < T ? bf16_bits_to_float(x[(size_t)tt * cols + col]) : 0.f;
        S.xp[i] = v * code_prescale(col & 7);
    }
    __syncthreads();
    stage_chunk_sums<NT>(S, kQgWarps);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (;;) {
        int rb = 0;
        if (lane == 0) rb = (int)atomicAdd(ctr, 1u);
        rb = __shfl_sync(0xffffffffu, rb, 0);
        if (rb >= nrb) break;
        const uint32_t *qq[1] = {q + (size_t)rb * C * 128};
        const uint32_t *ss[1] = {sb + (size_t)rb * G * 32};
        float acc[1][NT];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) acc[0][tt] = 0.f;
        gemv_slice<NT, 1>(qq, ss, S, T, 0, G, acc);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
            if (tt < T) y[(size_t)tt * rows + (size_t)rb * kRowBlock + lane] = acc[0][tt];
    }
}

size_t qmat_gemv_smem(int cols, int T) {
    const int nt = T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : 8));
    return stage_bytes(cols, nt, 0);
}

template <int NT>
static cudaError_t launch_qmat_gemv_nt(const moe_qmat &w, int rows, int cols, const uint16_t *x, int T, float *y,
                                       unsigned *ctr, cudaStream_t st) {
    const size_t smem = stage_bytes(cols, NT, 0);
    const void *fn = reinterpret_cast<const void *>(qmat_gemv_kernel<NT>);
    cudaError_t e = ensure_smem(fn, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per = 0;
    // the SM count of the device that runs the kernel
    if ((e = stream_device(st, &dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, kQgWarps * 32, smem)) != cudaSuccess) return e;
    const int nrb = rows / kRowBlock;
    int grid = sms * (per > 0 ? per : 1);
    if (grid * kQgWarps > nrb) grid = (nrb + kQgWarps - 1) / kQgWarps;
    if ((e = cudaMemsetAsync(ctr, 0, sizeof(unsigned), st)) != cudaSuccess) return e;
    qmat_gemv_kernel<NT><<<grid, kQgWarps * 32, smem, st>>>(w.q, w.sb, rows, cols, x, T, y, ctr);
    return cudaGetLastError();
}

cudaError_t launch_qmat_gemv(const moe_qmat &w, int rows, int cols, const uint16_t *x, int T, float *y,
                             unsigned *ctr, cudaStream_t st) {
    if (T <= 1) return launch_qmat_gemv_nt<1>(w, rows, cols, x, T, y, ctr, st);
    if (T <= 2) return launch_qmat_gemv_nt<2>(w, rows, cols, x, T, y, ctr, st);
    if (T <= 4) return launch_qmat_gemv_nt<4>(w, rows, cols, x, T, y, ctr, st);
    return launch_qmat_gemv_nt<8>(w, rows, cols, x, T, y, ctr, st);
}

cudaError_t launch_expert_gemv(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                               const int32_t *perm, const int32_t *active, int with_shared, const FfnBuffers &b,
                               cudaStream_t st) {
    ExpertParams P;
    P.gq = w->gate.q;
    P.gsb = w->gate.sb;
    P.uq = w->up.q;
    P.usb = w->up.sb;
    P.dq = w->down.q;
    P.dsb = w->down.sb;
    P.sgq = w->sh_gate.q;
    P.sgsb = w->sh_gate.sb;
    P.suq = w->sh_up.q;
    P.susb = w->sh_up.sb;
    P.sdq = w->sh_down.q;
    P.sdsb = w->sh_down.sb;
    P.xe = xe;
    P.offsets = offsets;
    P.perm = perm;
    P.active = active;
    P.a_routed = b.a_routed;
    P.a_shared = b.a_shared;
    P.y = b.y;
    P.sh = b.sh;
    P.T = T;
    P.H = w->H;
    P.I = w->I;
    P.Is = w->Is;
    P.k = w->k;
    P.with_shared = with_shared;
    long long pairs = (long long)T * w->k;
    const int max_active = (int)(pairs < w->E ? pairs : w->E);
    if (T == 1) return launch_ffn_nt<1>(P, max_active, st);
    return launch_ffn_nt<4>(P, max_active, st);
}

}  // namespace moe
