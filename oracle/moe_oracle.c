/*
 * moe_oracle.c -- plain, slow fp64 CPU oracle for one sparse Mixture-of-Experts
 * layer with MLX-affine quantised weights.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes, and where the pages say so (all on the TurboFieldfare
 * introduction page, discuss.pytorch.kr, unless noted):
 *   - router, section "TurboFieldfare's expert streaming structure", the
 *     router pseudo-code: rmsnorm_no_scale(hidden) -> * router_scale /
 *     sqrt(hidden_size) -> 8-bit affine projection -> highest k ->
 *     softmax(logits[topk]) * per_expert_scale[topk];
 *   - weight format, section "How TurboFieldfare saves memory": MLX affine,
 *     4-bit values in groups of 64 with a BF16 scale and a BF16 bias per
 *     group; only the router projection is 8-bit;
 *   - shared expert added without a routing weight, and the second command
 *     buffer (weighted sum of the routed branches + shared branch, then
 *     normalisation, residual and layer scalar), section "TurboFieldfare's
 *     expert streaming structure";
 *   - expert shapes (E, k): same section, and the Swiftlet article
 *     (tech.utomolab.com), section "Why the same model runs in so little
 *     memory".
 * Readings where the pages are silent (each also stated at its function):
 *   eps = 1e-6 inside the RMS; router_scale is a per-dimension vector; 8-bit
 *   codes are unsigned like MLX's 4-bit ones; top-k ties go to the lower
 *   expert index and the output is ordered by (logit desc, index asc); the
 *   per-expert scale is applied after the softmax with no renormalisation;
 *   experts consume bf16(rmsnorm_no_scale(h)); the expert activation is
 *   SwiGLU silu(g) * u; the post-combine normalisation is a weightless RMS
 *   norm, out = (h + rmsnorm_no_scale(m)) * layer_scalar; every conversion to
 *   bf16 rounds to nearest even, directly from fp64.
 *
 * Everything is fp64.  Dequantised weights are exact in fp64
 * (bf16 scale * small integer + bf16 bias).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL -1

/* Threads of the row loops (1 = the plain sequential oracle).  Returns the
 * count in effect: 1 when the library was built without OpenMP. */
int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n < 1) n = 1;
    omp_set_num_threads(n);
    return n;
#else
    (void)n;
    return 1;
#endif
}

/* ---------------------------------------------------------------- bf16 */

/* bf16 bit pattern -> double (exact: bf16 is the top half of an fp32). */
double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16 bits, round to nearest, ties to even, in one step from fp64.
 * bf16 keeps 8 significant bits and fp32's exponent range: the value is
 * scaled so that its last kept bit has weight 1, rounded with rint (the
 * default rounding mode is to nearest-even), and scaled back; all of that is
 * exact in fp64.  The result is then exactly representable in fp32. */
uint16_t oracle_double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    double ax = fabs(x);
    double y;
    if (ax == 0.0) {
        y = x;
    } else {
        int e;
        frexp(ax, &e);                 /* ax = m * 2^e, 0.5 <= m < 1 */
        int lsb = e - 8;               /* weight of the last kept bit (normal range) */
        if (lsb < -133) lsb = -133;    /* bf16 subnormal quantum is 2^-133 */
        y = ldexp(rint(ldexp(x, -lsb)), lsb);
        /* largest finite bf16 is (2 - 2^-7) * 2^127 */
        if (fabs(y) > ldexp(255.0, 120)) y = copysign(INFINITY, x);
    }
    float f = (float)y;                /* exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* --------------------------------------------------------- dequantisation */

/* Code of element `col` of a packed row: fields of `bits` bits, low field
 * first, 32/bits fields per uint32 word (MLX packing). */
static unsigned code_at(const uint32_t *row_words, int col, int bits)
{
    int per = 32 / bits;
    uint32_t w = row_words[col / per];
    return (w >> (bits * (col % per))) & ((1u << bits) - 1u);
}

/* w = scale * q + bias, with the scale/bias of group col/64 (MLX affine,
 * TurboFieldfare page, "How TurboFieldfare saves memory"). */
static double deq(const uint32_t *q, const uint16_t *s, const uint16_t *b, int cols, int bits,
                  int row, int col)
{
    const uint32_t *rw = q + (size_t)row * (size_t)(cols * bits / 32);
    int g = col / 64;
    size_t gi = (size_t)row * (size_t)(cols / 64) + (size_t)g;
    return oracle_bf16_to_double(s[gi]) * (double)code_at(rw, col, bits) + oracle_bf16_to_double(b[gi]);
}

/* Dequantise a whole [rows, cols] matrix into fp64 (used by tests). */
int oracle_dequant(const uint32_t *q, const uint16_t *s, const uint16_t *b, int rows, int cols, int bits,
                   double *out)
{
    if (cols % 64 || (bits != 4 && bits != 8)) return ORACLE_EINVAL;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            out[(size_t)r * cols + c] = deq(q, s, b, cols, bits, r, c);
    return ORACLE_OK;
}

/* y[r] = sum_c deq(W[r, c]) * x[c] : the affine-quantised projection.
 * Rows are independent and each row's sum runs in the same order whatever
 * the thread count, so the OpenMP split (when the library is built with it
 * and oracle_set_threads asks for more than one thread) changes nothing in
 * the result. */
static void qmatvec(const uint32_t *q, const uint16_t *s, const uint16_t *b, int rows, int cols, int bits,
                    const double *x, double *y)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(static) if ((long)rows * cols >= 65536)
#endif
    for (int r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int c = 0; c < cols; ++c) acc += deq(q, s, b, cols, bits, r, c) * x[c];
        y[r] = acc;
    }
}

/* Y[t][r] = sum_c deq(W[r, c]) * X[t][c] for T input rows: one quantised
 * matrix applied to T vectors, e.g. the vocabulary-sized output head that
 * shares the embedding's quantised weights (TurboFieldfare page, "How
 * TurboFieldfare saves memory"). */
int oracle_qmat_gemv(const uint32_t *q, const uint16_t *s, const uint16_t *b, int rows, int cols, int bits,
                     const double *x, int T, double *y)
{
    if (cols % 64 || (bits != 4 && bits != 8) || rows < 0 || T < 0) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) qmatvec(q, s, b, rows, cols, bits, x + (size_t)t * cols, y + (size_t)t * rows);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ router */

/* rmsnorm_no_scale (router pseudo-code, first line): xn = h / sqrt(mean(h^2) + eps).
 * No learned weight.  eps is not on the pages; 1e-6 is the reading used. */
void oracle_rmsnorm_no_scale(const double *h, int H, double eps, double *xn)
{
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += h[i] * h[i];
    double r = sqrt(ss / (double)H + eps);
    for (int i = 0; i < H; ++i) xn[i] = h[i] / r;
}

typedef struct {
    double v;
    int e;
} scored;

/* Highest logit first; equal logits -> lower expert index first. */
static int cmp_scored(const void *pa, const void *pb)
{
    const scored *a = (const scored *)pa, *b = (const scored *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->e > b->e) - (a->e < b->e);
}

/* highest_k (router pseudo-code, fourth line): full sort of (logit, index)
 * by logit descending then index ascending; the first k are the selection,
 * in that order. */
int oracle_topk(const double *logits, int E, int k, int32_t *idx)
{
    if (k < 1 || k > E) return ORACLE_EINVAL;
    scored *all = (scored *)malloc(sizeof(scored) * (size_t)E);
    if (!all) return ORACLE_EINVAL;
    for (int e = 0; e < E; ++e) {
        all[e].v = logits[e];
        all[e].e = e;
    }
    qsort(all, (size_t)E, sizeof(scored), cmp_scored);
    for (int s = 0; s < k; ++s) idx[s] = all[s].e;
    free(all);
    return ORACLE_OK;
}

/* weights = softmax(logits[topk]) * per_expert_scale[topk] (router
 * pseudo-code, last line).  The softmax runs over the k selected logits only,
 * max-subtracted; the per-expert scale is applied afterwards and the weights
 * are NOT renormalised.  p_out (optional) receives the softmax alone. */
void oracle_gate_weights(const double *logits, const int32_t *idx, int k, const uint16_t *per_expert_scale,
                         double *w, double *p_out)
{
    double mx = logits[idx[0]];
    for (int s = 1; s < k; ++s)
        if (logits[idx[s]] > mx) mx = logits[idx[s]];
    double z = 0.0;
    for (int s = 0; s < k; ++s) z += exp(logits[idx[s]] - mx);
    for (int s = 0; s < k; ++s) {
        double p = exp(logits[idx[s]] - mx) / z;
        if (p_out) p_out[s] = p;
        w[s] = p * oracle_bf16_to_double(per_expert_scale[idx[s]]);
    }
}

typedef struct {
    int H, E, k, I, Is;
    /* router: codes [E, H/4] (8-bit), scale/bias [E, H/64] */
    const uint32_t *router_q;
    const uint16_t *router_s, *router_b;
    const uint16_t *router_scale;      /* [H] */
    const uint16_t *per_expert_scale;  /* [E] */
    /* routed experts, stacked: gate/up [E, I, H/8], down [E, H, I/8]; groups [.., cols/64] */
    const uint32_t *gate_q, *up_q, *down_q;
    const uint16_t *gate_s, *gate_b, *up_s, *up_b, *down_s, *down_b;
    /* shared expert: gate/up [Is, H/8], down [H, Is/8] */
    const uint32_t *sh_gate_q, *sh_up_q, *sh_down_q;
    const uint16_t *sh_gate_s, *sh_gate_b, *sh_up_s, *sh_up_b, *sh_down_s, *sh_down_b;
} oracle_layer;

static int check_layer(const oracle_layer *L)
{
    if (!L || L->H % 64 || L->I % 64 || L->Is % 64 || L->k < 1 || L->k > L->E) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/* Router for T tokens.  h: [T, H] bf16 bits.  Outputs: logits [T, E] (may be
 * NULL), idx [T, k], w [T, k], xn [T, H] fp64 (may be NULL).
 *   xn = rmsnorm_no_scale(h)
 *   xs = xn * router_scale / sqrt(H)          (router_scale read as a [H] vector)
 *   logit_e = sum_i deq(R[e, i]) * xs_i       (8-bit affine, unsigned codes)
 */
int oracle_router(const oracle_layer *L, const uint16_t *h, int T, double eps, double *logits_out,
                  int32_t *idx, double *w, double *xn_out)
{
    if (check_layer(L) || T < 0) return ORACLE_EINVAL;
    int H = L->H, E = L->E, k = L->k;
    double *hd = (double *)malloc(sizeof(double) * (size_t)H);
    double *xn = (double *)malloc(sizeof(double) * (size_t)H);
    double *xs = (double *)malloc(sizeof(double) * (size_t)H);
    double *lg = (double *)malloc(sizeof(double) * (size_t)E);
    if (!hd || !xn || !xs || !lg) {
        free(hd); free(xn); free(xs); free(lg);
        return ORACLE_EINVAL;
    }
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < H; ++i) hd[i] = oracle_bf16_to_double(h[(size_t)t * H + i]);
        oracle_rmsnorm_no_scale(hd, H, eps, xn);
        for (int i = 0; i < H; ++i) xs[i] = xn[i] * oracle_bf16_to_double(L->router_scale[i]) / sqrt((double)H);
        qmatvec(L->router_q, L->router_s, L->router_b, E, H, 8, xs, lg);
        oracle_topk(lg, E, k, idx + (size_t)t * k);
        oracle_gate_weights(lg, idx + (size_t)t * k, k, L->per_expert_scale, w + (size_t)t * k, NULL);
        if (logits_out) memcpy(logits_out + (size_t)t * E, lg, sizeof(double) * (size_t)E);
        if (xn_out) memcpy(xn_out + (size_t)t * H, xn, sizeof(double) * (size_t)H);
    }
    free(hd); free(xn); free(xs); free(lg);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ bucket */

/* Token -> expert bucketing: count pairs per expert, exclusive scan into
 * offsets[E+1], and list pair ids p = t*k + s grouped by expert, within an
 * expert in ascending p (i.e. by token, then slot).  inv[perm[j]] = j.
 * (The pages' chunked prefill lets many rows share one fetched expert:
 * TurboFieldfare page, "expert streaming structure", last paragraph.) */
int oracle_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm, int32_t *inv)
{
    if (T < 0 || k < 1 || E < 1) return ORACLE_EINVAL;
    int n = T * k;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int p = 0; p < n; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return ORACLE_EINVAL;
        offsets[idx[p] + 1] += 1;
    }
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    if (!cursor) return ORACLE_EINVAL;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int p = 0; p < n; ++p) perm[cursor[idx[p]]++] = p;
    for (int j = 0; j < n; ++j) inv[perm[j]] = j;
    free(cursor);
    return ORACLE_OK;
}

/* ----------------------------------------------------------------- experts */

/* One SwiGLU expert applied to x [H] (the activation is not named on the
 * pages; SwiGLU is the reading):
 *   g = Wg x,  u = Wu x,  a = g * sigmoid(g) * u = g / (1 + exp(-g)) * u,  y = Wd a.
 * gq/gs/gb etc. point at this expert's matrices.  scratch: 3 * inter doubles. */
static void expert_ffn(int H, int inter, const uint32_t *gq, const uint16_t *gs, const uint16_t *gb,
                       const uint32_t *uq, const uint16_t *us, const uint16_t *ub, const uint32_t *dq,
                       const uint16_t *ds, const uint16_t *db, const double *x, double *y, double *scratch)
{
    double *g = scratch, *u = scratch + inter, *a = scratch + 2 * inter;
    qmatvec(gq, gs, gb, inter, H, 4, x, g);
    qmatvec(uq, us, ub, inter, H, 4, x, u);
    for (int j = 0; j < inter; ++j) a[j] = g[j] / (1.0 + exp(-g[j])) * u[j];
    qmatvec(dq, ds, db, H, inter, 4, a, y);
}

/* Public single-expert entry (tests): expert e of the stacked routed
 * matrices, or the shared expert when e < 0. */
int oracle_expert(const oracle_layer *L, int e, const double *x, double *y)
{
    if (check_layer(L) || e >= L->E) return ORACLE_EINVAL;
    int H = L->H;
    int inter = e < 0 ? L->Is : L->I;
    double *scratch = (double *)malloc(sizeof(double) * 3 * (size_t)inter);
    if (!scratch) return ORACLE_EINVAL;
    if (e < 0) {
        expert_ffn(H, inter, L->sh_gate_q, L->sh_gate_s, L->sh_gate_b, L->sh_up_q, L->sh_up_s, L->sh_up_b,
                   L->sh_down_q, L->sh_down_s, L->sh_down_b, x, y, scratch);
    } else {
        size_t gw = (size_t)e * L->I * (H / 8), gg = (size_t)e * L->I * (H / 64);
        size_t dw = (size_t)e * H * (L->I / 8), dg = (size_t)e * H * (L->I / 64);
        expert_ffn(H, inter, L->gate_q + gw, L->gate_s + gg, L->gate_b + gg, L->up_q + gw, L->up_s + gg,
                   L->up_b + gg, L->down_q + dw, L->down_s + dg, L->down_b + dg, x, y, scratch);
    }
    free(scratch);
    return ORACLE_OK;
}

/* Expert part of the layer for T tokens, straight from the definition (no
 * bucketing):  m_t = sum_s w[t,s] * FFN_{idx[t,s]}(x_t)  (+ FFN_shared(x_t)
 * with weight 1 when with_shared).  x: [T, H] fp64 (the experts' input);
 * m: [T, H]. */
int oracle_expert_ffn(const oracle_layer *L, const double *x, int T, const int32_t *idx, const double *w,
                      int with_shared, double *m)
{
    if (check_layer(L) || T < 0) return ORACLE_EINVAL;
    int H = L->H, k = L->k;
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    if (!y) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) {
        double *mt = m + (size_t)t * H;
        for (int o = 0; o < H; ++o) mt[o] = 0.0;
        for (int s = 0; s < k; ++s) {
            int e = idx[(size_t)t * k + s];
            if (e < 0 || e >= L->E) {
                free(y);
                return ORACLE_EINVAL;
            }
            oracle_expert(L, e, x + (size_t)t * H, y);
            for (int o = 0; o < H; ++o) mt[o] += w[(size_t)t * k + s] * y[o];
        }
        if (with_shared) {
            oracle_expert(L, -1, x + (size_t)t * H, y);
            for (int o = 0; o < H; ++o) mt[o] += y[o];
        }
    }
    free(y);
    return ORACLE_OK;
}

/* ----------------------------------------------------------------- combine */

/* Second command buffer tail: normalisation, residual, layer scalar, in that
 * order.  Reading: out = (h + rmsnorm_no_scale(m)) * layer_scalar when
 * post_norm, else (h + m) * layer_scalar.  out_f64 gets the exact value,
 * out_bf16 its round-to-nearest-even bf16. */
void oracle_combine(const uint16_t *h, const double *m, int T, int H, int post_norm, double layer_scalar,
                    double eps, double *out_f64, uint16_t *out_bf16)
{
    double *mn = (double *)malloc(sizeof(double) * (size_t)H);
    for (int t = 0; t < T; ++t) {
        const double *mt = m + (size_t)t * H;
        if (post_norm)
            oracle_rmsnorm_no_scale(mt, H, eps, mn);
        else
            memcpy(mn, mt, sizeof(double) * (size_t)H);
        for (int i = 0; i < H; ++i) {
            double v = (oracle_bf16_to_double(h[(size_t)t * H + i]) + mn[i]) * layer_scalar;
            if (out_f64) out_f64[(size_t)t * H + i] = v;
            if (out_bf16) out_bf16[(size_t)t * H + i] = oracle_double_to_bf16(v);
        }
    }
    free(mn);
}

/* ------------------------------------------------------------- whole layer */

/* One MoE layer on T tokens:
 *   router (idx, w, xn) -> experts consume xe = bf16(xn) -> m -> combine.
 * Outputs (each may be NULL): idx [T,k], w [T,k], m [T,H] fp64 (pre-norm
 * expert output), out_f64 [T,H], out_bf16 [T,H]. */
int oracle_layer_forward(const oracle_layer *L, const uint16_t *h, int T, double eps, int post_norm,
                         double layer_scalar, int32_t *idx_out, double *w_out, double *m_out,
                         double *out_f64, uint16_t *out_bf16)
{
    if (check_layer(L) || T < 0) return ORACLE_EINVAL;
    int H = L->H, k = L->k;
    size_t nT = (size_t)(T > 0 ? T : 1);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * nT * k);
    double *w = (double *)malloc(sizeof(double) * nT * k);
    double *xn = (double *)malloc(sizeof(double) * nT * H);
    double *m = (double *)malloc(sizeof(double) * nT * H);
    if (!idx || !w || !xn || !m) {
        free(idx); free(w); free(xn); free(m);
        return ORACLE_EINVAL;
    }
    int rc = oracle_router(L, h, T, eps, NULL, idx, w, xn);
    /* experts consume the router's normalised vector rounded to bf16 */
    for (size_t i = 0; rc == ORACLE_OK && i < (size_t)T * H; ++i)
        xn[i] = oracle_bf16_to_double(oracle_double_to_bf16(xn[i]));
    if (rc == ORACLE_OK) rc = oracle_expert_ffn(L, xn, T, idx, w, 1, m);
    if (rc == ORACLE_OK) {
        oracle_combine(h, m, T, H, post_norm, layer_scalar, eps, out_f64, out_bf16);
        if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)T * k);
        if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)T * k);
        if (m_out) memcpy(m_out, m, sizeof(double) * (size_t)T * H);
    }
    free(idx); free(w); free(xn); free(m);
    return rc;
}
