/*
 * moe_api.h -- C ABI of libmoe.so: one sparse Mixture-of-Experts layer with
 * MLX-affine quantised weights on NVIDIA B200 (sm_100a).
 *
 * The layer (TurboFieldfare introduction page, discuss.pytorch.kr, section
 * "TurboFieldfare's expert streaming structure", router pseudo-code and the
 * three-phase description; weight format from section "How TurboFieldfare
 * saves memory"):
 *   xn  = rmsnorm_no_scale(h)                       (no learned weight, eps inside the RMS)
 *   xs  = xn * router_scale / sqrt(H)
 *   logit_e = sum_i (s_e,g * q_e,i + b_e,g) * xs_i  (8-bit affine codes, groups of 64)
 *   idx = highest k logits (ties -> lower expert index; ordered by logit desc, index asc)
 *   w   = softmax(logit[idx]) * per_expert_scale[idx]   (no renormalisation)
 *   xe  = bf16(xn)                                  (what the experts consume)
 *   m   = sum_s w_s * FFN_idx_s(xe) + FFN_shared(xe) (shared expert: no routing weight)
 *   FFN(x) = Wd (silu(Wg x) * (Wu x)),  W = scale * q + bias, 4-bit codes, groups of 64
 *   out = (h + rmsnorm_no_scale(m)) * layer_scalar  (normalisation, residual, layer scalar)
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     16-byte aligned.  The library never allocates on these paths; scratch
 *     comes from a caller-provided workspace (see moe_workspace_size).
 *   - bf16 values are passed as their 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on that stream and returns; none synchronises.
 *   - Return value: MOE_OK (0) or a negative MOE_E* code.  Argument errors are
 *     detected on the host before anything is enqueued; the reason is then in
 *     moe_last_error() (per host thread).  Inputs are assumed finite.
 *   - T == 0 is a valid empty call: nothing is enqueued, MOE_OK is returned.
 *
 * Limits: H, I, Is multiples of 64 and <= 8192; 1 <= k <= min(E, 32);
 * E <= 1024 and a multiple of 8; 0 <= T <= 65535; T * k <= 65536.
 */
#ifndef MOE_API_H
#define MOE_API_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_EINVAL (-1)     /* bad size, null pointer, k > E, ... */
#define MOE_EALIGN (-2)     /* a pointer is not 16-byte aligned */
#define MOE_EWORKSPACE (-3) /* workspace missing or smaller than moe_workspace_size() */
#define MOE_ECUDA (-4)      /* a CUDA launch failed; the CUDA error string is in moe_last_error() */
#define MOE_EDEVICE (-5)    /* a kernel recorded an error (a bounded wait ran out); see moe_workspace_status */

/*
 * Quantised matrix set in the kernel ("tiled") layout, produced once per
 * weight tensor by moe_prepare_qmat from the MLX layout.  n_mat matrices of
 * [rows, cols] (rows % 32 == 0, cols % 64 == 0):
 *   q : uint32 words.  For matrix m, row block rb = row / 32, column chunk
 *       c = col / 32: a 512-byte block at word offset
 *       ((m * rows/32 + rb) * cols/32 + c) * 128; inside it, lane l = row % 32
 *       holds 4 consecutive words (the row's MLX words 4c .. 4c+3, i.e.
 *       columns 32c .. 32c+31, eight 4-bit codes per word, low nibble first).
 *   sb: uint32 per (matrix, row, group of 64 columns): low 16 bits = bf16
 *       scale, high 16 bits = bf16 bias; for matrix m, row block rb, group g,
 *       lane l at word offset ((m * rows/32 + rb) * cols/64 + g) * 32 + l.
 * One row block of one matrix is therefore contiguous, so a warp whose lanes
 * are 32 consecutive rows reads 512 contiguous bytes per column chunk.
 */
typedef struct {
    const uint32_t *q;
    const uint32_t *sb;
} moe_qmat;

/* One MoE layer's weights, all device pointers. */
typedef struct {
    int H;  /* hidden size */
    int E;  /* routed experts */
    int k;  /* experts per token */
    int I;  /* routed expert intermediate size */
    int Is; /* shared expert intermediate size */
    /* router projection, MLX layout: codes [E, H/4] (four 8-bit codes per word,
     * low byte first), bf16 scale and bias [E, H/64] */
    const uint32_t *router_q;
    const uint16_t *router_s;
    const uint16_t *router_b;
    const uint16_t *router_scale;     /* [H] bf16 */
    const uint16_t *per_expert_scale; /* [E] bf16 */
    /* routed experts, tiled layout: gate/up are E matrices [I, H], down E x [H, I] */
    moe_qmat gate, up, down;
    /* shared expert, tiled layout: gate/up [Is, H], down [H, Is] */
    moe_qmat sh_gate, sh_up, sh_down;
} moe_layer_w;

typedef struct {
    int post_norm;      /* 1: out = (h + rmsnorm_no_scale(m)) * layer_scalar; 0: (h + m) * layer_scalar */
    float layer_scalar; /* default 1.0 */
    float eps;          /* default 1e-6, inside every RMS */
    int force_path;     /* 0 auto: dequant-GEMV below 32 tokens, the weight-stationary warp-level MMA
                           for 32..448, the tcgen05 grouped GEMM above;
                           1 CUDA-core dequant-GEMV, 2 tensor-core (tcgen05) grouped GEMM,
                           3 weight-stationary warp-level MMA (exact codes, FP32 scale/bias) */
} moe_opts;

/* Text of the last error on this host thread ("" if none). */
MOE_API const char *moe_last_error(void);

/* Library version string. */
MOE_API const char *moe_version(void);

/*
 * Repack n_mat MLX-layout matrices [rows, cols] (codes q [n_mat, rows, cols/8]
 * uint32, scale/bias [n_mat, rows, cols/64] bf16) into the tiled layout
 * described at moe_qmat.  q_out has the same number of words as q;
 * sb_out has n_mat * rows * cols/64 words.  Off the hot path; done once per
 * weight tensor.  rows % 32 == 0, cols % 64 == 0.
 */
MOE_API int moe_prepare_qmat(const uint32_t *q, const uint16_t *scale, const uint16_t *bias, int n_mat, int rows,
                     int cols, uint32_t *q_out, uint32_t *sb_out, void *stream);

/*
 * Bytes of workspace that moe_router / moe_expert_ffn / moe_layer_forward
 * need for calls with up to T_max tokens on layers shaped like `w`.
 * Returns 0 on invalid arguments.  (The pages define no workspace: it is this
 * library's ownership rule -- the caller allocates every buffer, the calls
 * never allocate, so that they can be enqueued from code that may not
 * allocate.)  Layout and contents are private to the library; the first 16
 * bytes hold the status word that moe_workspace_status reads.
 */
MOE_API size_t moe_workspace_size(const moe_layer_w *w, int T_max);

/*
 * Synchronous: waits for the device, then reads the status word that the
 * last moe_expert_ffn / moe_layer_forward call on the tensor-core path left in
 * `ws` (its first bytes; reset by every such call).  The grouped-GEMM kernels
 * bound every wait (~1 s); if one runs out they record a code there and stop
 * early (outputs are then invalid).  MOE_OK, or MOE_EDEVICE with the reason in
 * moe_last_error().  Also reads a moe_decode_stack workspace.
 */
MOE_API int moe_workspace_status(const void *ws);

/*
 * Router logits only (the first three lines of the router pseudo-code):
 *   h [T, H] bf16  ->  logits [T, E] fp64, and (if xe != NULL) xe [T, H] bf16.
 * Accumulates in fp64 so that the top-k decision does not depend on the
 * summation order.
 */
MOE_API int moe_router_logits(const moe_layer_w *w, const uint16_t *h, int T, double *logits, uint16_t *xe,
                      void *stream);

/*
 * Top-k + gate weights (last two lines of the router pseudo-code):
 *   logits [T, E] fp64 -> idx [T, k] int32 (logit desc, index asc; equal
 *   logits -> lower index), wts [T, k] fp32 = softmax over the k selected
 *   logits * per_expert_scale[idx].
 */
MOE_API int moe_router_topk(const double *logits, int T, int E, int k, const uint16_t *per_expert_scale, int32_t *idx,
                    float *wts, void *stream);

/*
 * Whole router: h [T, H] bf16 -> idx [T, k], wts [T, k], xe [T, H] bf16 (xe
 * may be NULL).  Uses T * E * 8 bytes of the workspace for the logits.
 */
MOE_API int moe_router(const moe_layer_w *w, const uint16_t *h, int T, int32_t *idx, float *wts, uint16_t *xe,
               void *ws, size_t ws_bytes, void *stream);

/*
 * Token -> expert bucketing of the T*k (token, slot) pairs (TurboFieldfare
 * introduction page, section "TurboFieldfare's expert streaming structure",
 * last paragraph: prefill runs in chunks of up to 128 tokens so that several
 * rows share one read of an expert; grouping the pairs by expert is what
 * lets an expert's weights be read once for all of its rows):
 *   offsets [E+1]: exclusive prefix sum of pairs per expert;
 *   perm [T*k]   : pair ids p = t*k + s grouped by expert, ascending p inside
 *                  an expert (stable);
 *   inv [T*k]    : inv[perm[j]] = j (may be NULL);
 *   active [E+1] : active[0] = number of experts with at least one pair,
 *                  active[1..] = those experts ascending (may be NULL).
 * idx values must lie in [0, E); T * k <= 65536.
 */
MOE_API int moe_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm, int32_t *inv,
               int32_t *active, void *stream);

/*
 * Expert part of the layer: m [T, H] fp32 = sum_s wts[t,s] * FFN_idx[t,s](xe_t)
 * (+ FFN_shared(xe_t) when with_shared).  Inputs: xe [T, H] bf16, idx/wts
 * [T, k], and the bucketing of idx (offsets, perm, active from moe_bucket).
 * (TurboFieldfare introduction page, section "TurboFieldfare's expert
 * streaming structure": the routed experts' outputs are summed with the
 * router's weights and the shared expert's output is added without one;
 * weights are MLX affine 4-bit, groups of 64, a BF16 scale and bias per
 * group, section "How TurboFieldfare saves memory".)
 * Path: force_path 1, or T < 32 in auto mode, is the CUDA-core dequant-GEMV
 * (fp32 sums of exact products).  force_path 2, or T > 448 in auto mode, is the tcgen05
 * grouped GEMM on FP16 operands: it needs every weight s*q + b and every
 * SwiGLU value within the FP16 range (|v| <= 65504).  A layer outside that
 * range is not computed approximately: the kernel records MOE_EDEVICE
 * ("outside the FP16 range") in the workspace status word (read it with
 * moe_workspace_status) and its outputs are invalid; use force_path 1 or 3 there.
 * force_path 3 runs the experts on the warp-level tensor cores with every
 * weight read once per group of 8 (gate/up) or 16 (down) tokens of an expert:
 * codes enter as exact FP16 values, scale and bias stay FP32, so only the
 * token rows and SwiGLU outputs are FP16 (a SwiGLU value beyond 65504 is
 * reported as above; weights have no range limit).  E <= 1024.  Auto mode takes
 * it for 32 <= T <= 448.
 */
MOE_API int moe_expert_ffn(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *idx, const float *wts,
                   const int32_t *offsets, const int32_t *perm, const int32_t *active, int with_shared,
                   float *m_out, void *ws, size_t ws_bytes, const moe_opts *opts, void *stream);

/*
 * One whole MoE layer: router -> bucketing -> routed + shared experts ->
 * weighted combine -> normalisation, residual, layer scalar (TurboFieldfare
 * introduction page, section "TurboFieldfare's expert streaming structure":
 * the router pseudo-code, then the three phases of a layer, the last of which
 * combines the routed branches with the router's weights, adds the shared
 * branch and applies normalisation, residual and the layer scalar).
 *   h_in [T, H] bf16 -> h_out [T, H] bf16 (h_out may not alias h_in).
 * opts may be NULL (post_norm 1, layer_scalar 1, eps 1e-6, auto path).  The
 * expert part follows the path rules of moe_expert_ffn.
 */
MOE_API int moe_layer_forward(const moe_layer_w *w, const uint16_t *h_in, uint16_t *h_out, int T, void *ws,
                      size_t ws_bytes, const moe_opts *opts, void *stream);

/*
 * Tiered expert residency: a layer whose routed experts live in a pool in
 * host memory, with a cache of `slots` experts in device memory
 * (TurboFieldfare introduction page, section "TurboFieldfare's expert
 * streaming structure": a 16-slot LFU cache of experts per layer, and only
 * the misses are read; Swiftlet article, section "why the same model runs in
 * so little memory": an LFU + recency cache pool).  The pool is the routed
 * gate/up/down matrices of all E experts in the tiled layout (as in
 * moe_layer_w), in pinned host memory that the GPU can address (cudaHostAlloc,
 * or torch's pin_memory); the cache has the same layout for `slots` experts
 * in device memory.  The bookkeeping arrays are device memory owned by the
 * caller and set up once by moe_expert_cache_reset.
 */
typedef struct {
    int slots;                              /* C >= the distinct experts one call can select: min(E, T*k) */
    moe_qmat gate, up, down;                /* device cache, C experts */
    moe_qmat pool_gate, pool_up, pool_down; /* host pool, E experts (device-addressable pinned memory) */
    int32_t *slot_of;                       /* [E]: cache slot of expert e, -1 when not resident */
    int32_t *expert_of;                     /* [C]: expert in slot s, -1 when empty */
    uint32_t *uses;                         /* [C]: uses of the slot's expert since it was loaded */
    uint32_t *last;                         /* [C]: the call that last used the slot */
    uint32_t *ctl;                          /* [4]: calls, hits, misses (cumulative; distinct experts per call), spare */
} moe_expert_cache;

/* Empties the cache (every slot free, counters 0).  E: the layer's routed experts. */
MOE_API int moe_expert_cache_reset(const moe_expert_cache *c, int E, void *stream);

/*
 * moe_layer_forward with the routed experts served from a cache.  w supplies
 * the router, the per-expert scales and the shared expert (resident); its
 * routed gate/up/down pointers are not used.  Per call, on the GPU: the
 * router; then, for the distinct experts selected, in ascending expert
 * order: a resident expert counts a use; a missing one takes the slot with
 * the fewest uses among those this call does not need (an empty slot first;
 * ties: least recently used, then the lowest slot) and is copied from the
 * pool over the bus; then bucketing, the experts (on the cache, by slot) and
 * the combine.  The result equals moe_layer_forward's on the same weights.
 * Workspace: moe_workspace_size(w, T).  Asynchronous; MOE_EINVAL when
 * slots < min(E, T*k).
 */
MOE_API int moe_layer_forward_cached(const moe_layer_w *w, const moe_expert_cache *c, const uint16_t *h_in,
                                     uint16_t *h_out, int T, void *ws, size_t ws_bytes, const moe_opts *opts,
                                     void *stream);

/*
 * Expert-parallel split of a layer over G devices (no counterpart in the
 * pages, which run one device; the split is this library's multi-GPU form of
 * the same arithmetic).  A rank owns the routed experts [e_lo, e_hi) --
 * contiguous blocks, e.g. [E*r/G, E*(r+1)/G) -- and, when with_shared != 0,
 * the shared expert (one rank per layer).  Every rank runs the whole router
 * (it is small) and computes
 *   m_out [T, H] fp32 = sum over its pairs of w_s * FFN_idx_s(xe)  (+ FFN_shared(xe)),
 * so that the sum of every rank's m_out is moe_expert_ffn's m for the layer
 * (up to fp32 summation order).  The caller adds the ranks' m_out (an
 * all-reduce, e.g. NCCL over NVLink) and finishes the layer with moe_combine.
 *   h_in [T, H] bf16; ws: moe_workspace_size(w, T) bytes.  Asynchronous; the
 *   expert part follows the path rules of moe_expert_ffn.
 */
MOE_API int moe_layer_partial(const moe_layer_w *w, const uint16_t *h_in, int T, int e_lo, int e_hi, int with_shared,
                              float *m_out, void *ws, size_t ws_bytes, const moe_opts *opts, void *stream);

/*
 * The end of a layer (TurboFieldfare introduction page, section
 * "TurboFieldfare's expert streaming structure": after the weighted combine,
 * normalisation, residual and layer scalar):
 *   h_out [T, H] bf16 = bf16((h_in + rmsnorm_no_scale(m)) * layer_scalar)   (post_norm, else h_in + m)
 * m [T, H] fp32 is the combine (e.g. the all-reduced sum of moe_layer_partial
 * outputs).  H a multiple of 64, <= 8192.  Asynchronous.
 */
MOE_API int moe_combine(const uint16_t *h_in, const float *m, uint16_t *h_out, int T, int H, const moe_opts *opts,
                        void *stream);

/*
 * Decode step through a stack of L layers (the per-token layer loop of the
 * TurboFieldfare page, section "TurboFieldfare's expert streaming structure",
 * last paragraph) in ONE persistent cooperative kernel, one CTA per SM.  Per
 * layer it computes exactly what moe_layer_forward computes.
 *   layers [L]  : HOST array of L layer descriptors, all with the same shape
 *                 (its contents are copied into the launch; L <= 64).
 *   h_in        : chained != 0: [T, H], the input of layer 0;
 *                 chained == 0: [L, T, H], layer l's own input.
 *   h_out [L,T,H]: every layer's output (chained: layer l's output is layer
 *                 l+1's input).
 *   1 <= T <= 8, H <= 4096, T * H <= 24576.  Needs cooperative launch.
 * opts->force_path picks how the experts' dot products run: 1 CUDA-core FMAs
 * (exact products, fp32 sums), 2 the warp-level tensor cores (BF16 operands:
 * codes as exact 128 + q, expert inputs as BF16 -- exact for gate/up, a
 * high + low pair for down -- fp32 accumulation; 3 means the same here), 0
 * automatic: CUDA cores for T = 1, tensor cores for T >= 2 (the FMA work grows
 * with T, the MMA's does not).
 * The first call with a given layer array encodes TMA descriptors on the host
 * (cached), and every call copies them into the workspace before the kernel.
 * The workspace (moe_decode_stack_workspace_size) must stay untouched until
 * the kernel finishes; its first bytes are reset by every call.  Every wait in
 * the kernel is bounded (~1 s); if one runs out the kernel records a code in
 * the workspace and returns early (outputs are then invalid) -- read it with
 * moe_decode_stack_status.
 */
MOE_API size_t moe_decode_stack_workspace_size(const moe_layer_w *w, int T);

MOE_API int moe_decode_stack(const moe_layer_w *layers, int L, const uint16_t *h_in, int chained, uint16_t *h_out,
                             int T, void *ws, size_t ws_bytes, const moe_opts *opts, void *stream);

/* 1 if moe_decode_stack can run layers shaped like `w` with T tokens on the
 * stream's device (NULL: the current device) with the automatic path -- its
 * plan of shared memory and work per CTA fits one CTA per SM -- else 0 (also
 * on bad arguments).  Callers fall back to moe_layer_forward per layer when
 * it returns 0.  (A forced path that does not fit makes moe_decode_stack
 * return MOE_EINVAL.) */
MOE_API int moe_decode_stack_fits(const moe_layer_w *w, int T, void *stream);

/* Synchronous: reads the device error code a moe_decode_stack call left in
 * `ws` (after waiting for the device).  MOE_OK, or MOE_EDEVICE with the reason
 * in moe_last_error(). */
MOE_API int moe_decode_stack_status(const void *ws);

/*
 * y[t][r] = sum_c W[r][c] * x[t][c] for ONE 4-bit MLX-affine matrix W
 * [rows, cols] in the tiled layout (moe_prepare_qmat with n_mat = 1), e.g. the
 * vocabulary-sized output head that shares the embedding's quantised weights
 * (TurboFieldfare introduction page, section "How TurboFieldfare saves
 * memory": embedding and language-model head share one quantised weight; the
 * decode-time table there lists that head at 14.2 ms of a 162.8 ms step).
 *   w        : device pointers q (codes) and sb (scale | bias << 16 words).
 *   rows     : a positive multiple of 32 (the vocabulary size for a head).
 *   cols     : a multiple of 64 in [64, 8192] (the hidden size).
 *   x [T, cols] bf16, y [T, rows] fp32, 1 <= T <= 8, all device, 16-byte aligned.
 *   ws       : moe_qmat_gemv_workspace_size() bytes of device memory, 16-byte
 *              aligned; the call resets it (a work counter); calls that overlap
 *              on the GPU need workspaces of their own.
 * Each weight group's products are exact (the code times the pre-scaled input)
 * and accumulate in fp32.  Asynchronous on `stream`; MOE_EINVAL / MOE_EALIGN /
 * MOE_EWORKSPACE on bad arguments, MOE_ECUDA on a launch failure.
 */
MOE_API size_t moe_qmat_gemv_workspace_size(void);

MOE_API int moe_qmat_gemv(const moe_qmat *w, int rows, int cols, const uint16_t *x, int T, float *y, void *ws,
                          size_t ws_bytes, void *stream);

/*
 * moe_layer_forward for callers that cannot allocate device memory.  (The
 * pages have no counterpart: this is a deployment convenience.)
 *
 * Some callers cannot call cudaMalloc on this path: code that runs while a
 * stream is being captured into a CUDA graph in the global capture mode
 * (allocation is forbidden there), latency-critical serving loops where an
 * allocation may synchronise the device, and plugins that run inside a host
 * framework that owns all device memory.  This entry point takes the same
 * arguments as moe_layer_forward minus the workspace, and uses instead a
 * scratch array of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) that the library
 * defines in device memory; every GPU that loads the library holds that array
 * until the process exits.  It calls no cudaMalloc, cudaFree or allocating
 * library routine.
 *   - Sizes whose workspace (moe_workspace_size) exceeds the scratch are
 *     rejected with MOE_EWORKSPACE and a message naming both sizes; decode
 *     batches fit (about 140 KiB per token at hidden 2816, 128 experts, top-8).
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins.  The device is the stream's device
 *     (the current device for the NULL stream).
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; nothing in it needs to start at zero.  Calls whose
 *     kernels overlap on the GPU (different streams, or several host threads)
 *     race on the scratch: serialise them.
 *   - The looked-up address is kept for the life of the process.  It does not
 *     survive cudaDeviceReset (or any other teardown of the device's primary
 *     context): do not call this entry point after one.
 *   - The tensor-core paths (T >= 32, or force_path 2 or 3) leave their status words
 *     in the scratch; moe_noalloc_status reads them.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

MOE_API size_t moe_noalloc_scratch_bytes(void);

MOE_API int moe_layer_forward_noalloc(const moe_layer_w *w, const uint16_t *h_in, uint16_t *h_out, int T,
                                      const moe_opts *opts, void *stream);

/*
 * Synchronous: waits for `stream` (the NULL stream: the current device), then
 * reads the status words that the last moe_layer_forward_noalloc call on the
 * stream's device left in the static scratch -- what moe_workspace_status
 * reads for a caller-provided workspace: MOE_OK, or MOE_EDEVICE with the
 * reason (a bounded wait that ran out, or a value outside the FP16 range of
 * the tensor-core path) in moe_last_error().  Allocates nothing.
 */
MOE_API int moe_noalloc_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_API_H */
