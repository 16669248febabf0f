// moe_api.cu -- the C ABI of libmoe.so: argument checks, workspace carving,
// and the launch sequence of each call.  See include/moe_api.h.
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <unordered_map>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

cudaError_t ensure_smem(const void *kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    static std::mutex mu;
    static std::unordered_map<const void *, size_t> done;
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(kernel);
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done[kernel] = bytes;
    return e;
}

}  // namespace moe

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *where) {
    return fail(MOE_ECUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDim = 8192;
constexpr int kMaxT = 65535;

#define CHECK_PTR(p)                                                                 \
    do {                                                                             \
        if (!(p)) return fail(MOE_EINVAL, "%s: %s is NULL", fn, #p);                 \
        if (!aligned16(p)) return fail(MOE_EALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
    } while (0)

#define CHECK_OPT_PTR(p)                                                             \
    do {                                                                             \
        if ((p) && !aligned16(p)) return fail(MOE_EALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
    } while (0)

int check_dims(const char *fn, const moe_layer_w *w) {
    if (!w) return fail(MOE_EINVAL, "%s: layer is NULL", fn);
    if (w->H < 64 || w->H % 64 || w->H > kMaxDim) return fail(MOE_EINVAL, "%s: H=%d must be a multiple of 64 in [64, %d]", fn, w->H, kMaxDim);
    if (w->I < 64 || w->I % 64 || w->I > kMaxDim) return fail(MOE_EINVAL, "%s: I=%d must be a multiple of 64 in [64, %d]", fn, w->I, kMaxDim);
    if (w->Is < 64 || w->Is % 64 || w->Is > kMaxDim) return fail(MOE_EINVAL, "%s: Is=%d must be a multiple of 64 in [64, %d]", fn, w->Is, kMaxDim);
    if (w->E < 8 || w->E % 8 || w->E > moe::kMaxE) return fail(MOE_EINVAL, "%s: E=%d must be a multiple of 8 in [8, %d]", fn, w->E, moe::kMaxE);
    if (w->k < 1 || w->k > w->E || w->k > moe::kMaxK) return fail(MOE_EINVAL, "%s: k=%d must be in [1, min(E, %d)]", fn, w->k, moe::kMaxK);
    return MOE_OK;
}

int check_router_ptrs(const char *fn, const moe_layer_w *w) {
    CHECK_PTR(w->router_q);
    CHECK_PTR(w->router_s);
    CHECK_PTR(w->router_b);
    CHECK_PTR(w->router_scale);
    CHECK_PTR(w->per_expert_scale);
    return MOE_OK;
}

int check_expert_ptrs(const char *fn, const moe_layer_w *w, int with_shared) {
    CHECK_PTR(w->gate.q);
    CHECK_PTR(w->gate.sb);
    CHECK_PTR(w->up.q);
    CHECK_PTR(w->up.sb);
    CHECK_PTR(w->down.q);
    CHECK_PTR(w->down.sb);
    if (with_shared) {
        CHECK_PTR(w->sh_gate.q);
        CHECK_PTR(w->sh_gate.sb);
        CHECK_PTR(w->sh_up.q);
        CHECK_PTR(w->sh_up.sb);
        CHECK_PTR(w->sh_down.q);
        CHECK_PTR(w->sh_down.sb);
    }
    return MOE_OK;
}

int check_T(const char *fn, int T) {
    if (T < 0 || T > kMaxT) return fail(MOE_EINVAL, "%s: T=%d must be in [0, %d]", fn, T, kMaxT);
    return MOE_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace carve-up for calls of up to T tokens.  The first 256 bytes hold
// the device status word (byte offset 4, as in the decode-stack workspace).
// The SwiGLU buffers of the GEMV path and the token / SwiGLU matrices of the
// tensor-core path share one region (a call uses one path).
struct WsLayout {
    size_t status, logits, idx, wts, xe, offsets, perm, inv, active, wts_ep, active_ep, idx_c, miss, a_routed,
        a_shared, xg, act, y, sh, total;
};

constexpr size_t kStatusOffset = 4;
constexpr int kMmaMinT = 32;   // auto path: tensor cores from this many tokens on (else the dequant-GEMV)
constexpr int kWsMaxT = 448;   // ... the weight-stationary warp-MMA path up to this many, the tcgen05 GEMM above
                               // (measured on the Gemma shape: the warp-MMA path ahead up to 448 tokens)

WsLayout ws_layout(const moe_layer_w *w, int T) {
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t Tk = (size_t)T * w->k;
    L.status = take(256);
    L.logits = take(sizeof(double) * T * w->E);
    L.idx = take(sizeof(int32_t) * Tk);
    L.wts = take(sizeof(float) * Tk);
    L.xe = take(sizeof(uint16_t) * T * w->H);
    L.offsets = take(sizeof(int32_t) * (w->E + 1));
    L.perm = take(sizeof(int32_t) * Tk);
    L.inv = take(sizeof(int32_t) * Tk);
    L.active = take(sizeof(int32_t) * (w->E + 1));
    L.wts_ep = take(sizeof(float) * Tk);
    L.active_ep = take(sizeof(int32_t) * (w->E + 1));
    L.idx_c = take(sizeof(int32_t) * Tk);
    L.miss = take(sizeof(int32_t) * (2 * (size_t)w->E + 1));
    {
        const size_t gemv_a = align256(sizeof(float) * Tk * w->I), gemv_s = align256(sizeof(float) * T * w->Is);
        const size_t mma_x = align256(moe::mma_xg_bytes(w, T)), mma_a = align256(moe::mma_act_bytes(w, T));
        const size_t region = take(gemv_a + gemv_s > mma_x + mma_a ? gemv_a + gemv_s : mma_x + mma_a);
        L.a_routed = region;
        L.a_shared = region + gemv_a;
        L.xg = region;
        L.act = region + mma_x;
    }
    L.y = take(sizeof(float) * Tk * w->H);
    L.sh = take(sizeof(float) * T * w->H);
    L.total = off;
    return L;
}

template <typename P>
P *at(void *ws, size_t off) {
    return reinterpret_cast<P *>(static_cast<char *>(ws) + off);
}

int check_ws(const char *fn, const moe_layer_w *w, int T, void *ws, size_t ws_bytes) {
    const size_t need = ws_layout(w, T).total;
    if (!ws) return fail(MOE_EWORKSPACE, "%s: workspace is NULL (need %zu bytes)", fn, need);
    if (!aligned16(ws)) return fail(MOE_EALIGN, "%s: workspace is not 16-byte aligned", fn);
    if (ws_bytes < need) return fail(MOE_EWORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn, ws_bytes, need);
    return MOE_OK;
}

moe_opts resolve_opts(const moe_opts *o) {
    moe_opts r{1, 1.0f, 1e-6f, 0};
    if (o) r = *o;
    return r;
}

int check_opts(const char *fn, const moe_opts &o) {
    if (o.force_path < 0 || o.force_path > 3)
        return fail(MOE_EINVAL, "%s: force_path=%d (0 auto, 1 dequant-GEMV, 2 tcgen05 grouped GEMM, 3 warp-MMA "
                    "weight-stationary)", fn, o.force_path);
    if (!(o.eps >= 0.0f)) return fail(MOE_EINVAL, "%s: eps must be >= 0", fn);
    return MOE_OK;
}

enum Path { kPathGemv = 1, kPathTc = 2, kPathWs = 3 };

Path expert_path(const moe_opts &o, int T) {
    if (o.force_path != 0) return static_cast<Path>(o.force_path);
    if (T < kMmaMinT) return kPathGemv;
    return T <= kWsMaxT ? kPathWs : kPathTc;
}

// Expert part of a call: the SwiGLU FFNs of the routed and shared experts into
// y / sh, by the tensor-core grouped GEMM or the CUDA-core dequant-GEMV.
cudaError_t run_experts(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets, const int32_t *perm,
                        const int32_t *active, int with_shared, void *ws, const WsLayout &L, const moe_opts &o,
                        cudaStream_t st) {
    const Path path = expert_path(o, T);
    // the status words describe this call, whatever path it takes: timeout word, FP16-range word
    int *err = at<int>(ws, L.status + kStatusOffset);
    cudaError_t e = cudaMemsetAsync(err, 0, 2 * sizeof(int), st);
    if (e != cudaSuccess) return e;
    if (path != kPathGemv) {
        moe::MmaBuffers b{at<uint16_t>(ws, L.xg), at<uint16_t>(ws, L.act), at<float>(ws, L.y), at<float>(ws, L.sh), err,
                          err + 1};
        if (path == kPathWs) return moe::launch_expert_wsmma(w, xe, T, offsets, perm, active, with_shared, b, st);
        return moe::launch_expert_mma(w, xe, T, offsets, perm, active, with_shared, b, st);
    }
    moe::FfnBuffers b{at<float>(ws, L.a_routed), at<float>(ws, L.a_shared), at<float>(ws, L.y), at<float>(ws, L.sh)};
    return moe::launch_expert_gemv(w, xe, T, offsets, perm, active, with_shared, b, st);
}

}  // namespace

namespace moe {
int set_last_error(int code, const char *msg) { return fail(code, "%s", msg); }
}  // namespace moe

extern "C" {

const char *moe_last_error(void) { return g_err.c_str(); }

const char *moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

int moe_prepare_qmat(const uint32_t *q, const uint16_t *scale, const uint16_t *bias, int n_mat, int rows, int cols,
                     uint32_t *q_out, uint32_t *sb_out, void *stream) {
    const char *fn = "moe_prepare_qmat";
    g_err.clear();
    if (n_mat < 1 || rows < 32 || rows % 32 || cols < 64 || cols % 64 || rows > (1 << 20) || cols > kMaxDim)
        return fail(MOE_EINVAL, "%s: need n_mat >= 1, rows %% 32 == 0, cols %% 64 == 0 (got %d, %d, %d)", fn, n_mat,
                    rows, cols);
    CHECK_PTR(q);
    CHECK_PTR(scale);
    CHECK_PTR(bias);
    CHECK_PTR(q_out);
    CHECK_PTR(sb_out);
    cudaError_t e = moe::launch_prepare_qmat(q, scale, bias, n_mat, rows, cols, q_out, sb_out,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

size_t moe_workspace_size(const moe_layer_w *w, int T_max) {
    if (check_dims("moe_workspace_size", w) || T_max < 0 || T_max > kMaxT) return 0;
    return ws_layout(w, T_max).total;
}

int moe_router_logits(const moe_layer_w *w, const uint16_t *h, int T, double *logits, uint16_t *xe, void *stream) {
    const char *fn = "moe_router_logits";
    g_err.clear();
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if (int rc = check_router_ptrs(fn, w)) return rc;
    CHECK_PTR(h);
    CHECK_PTR(logits);
    CHECK_OPT_PTR(xe);
    if (T == 0) return MOE_OK;
    cudaError_t e = moe::launch_router_logits(w, h, T, 1e-6f, logits, xe, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_router_topk(const double *logits, int T, int E, int k, const uint16_t *per_expert_scale, int32_t *idx,
                    float *wts, void *stream) {
    const char *fn = "moe_router_topk";
    g_err.clear();
    if (int rc = check_T(fn, T)) return rc;
    if (E < 1 || E > moe::kMaxE) return fail(MOE_EINVAL, "%s: E=%d must be in [1, %d]", fn, E, moe::kMaxE);
    if (k < 1 || k > E || k > moe::kMaxK) return fail(MOE_EINVAL, "%s: k=%d must be in [1, min(E, %d)]", fn, k, moe::kMaxK);
    CHECK_PTR(logits);
    CHECK_PTR(per_expert_scale);
    CHECK_PTR(idx);
    CHECK_PTR(wts);
    if (T == 0) return MOE_OK;
    cudaError_t e = moe::launch_router_topk(logits, T, E, k, per_expert_scale, idx, wts,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_router(const moe_layer_w *w, const uint16_t *h, int T, int32_t *idx, float *wts, uint16_t *xe, void *ws,
               size_t ws_bytes, void *stream) {
    const char *fn = "moe_router";
    g_err.clear();
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if (int rc = check_router_ptrs(fn, w)) return rc;
    CHECK_PTR(h);
    CHECK_PTR(idx);
    CHECK_PTR(wts);
    CHECK_OPT_PTR(xe);
    if (T == 0) return MOE_OK;
    if (int rc = check_ws(fn, w, T, ws, ws_bytes)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(w, T);
    double *logits = at<double>(ws, L.logits);
    cudaError_t e = moe::launch_router_logits(w, h, T, 1e-6f, logits, xe, st);
    if (e == cudaSuccess) e = moe::launch_router_topk(logits, T, w->E, w->k, w->per_expert_scale, idx, wts, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_bucket(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm, int32_t *inv,
               int32_t *active, void *stream) {
    const char *fn = "moe_bucket";
    g_err.clear();
    if (int rc = check_T(fn, T)) return rc;
    if (E < 1 || E > moe::kMaxE) return fail(MOE_EINVAL, "%s: E=%d must be in [1, %d]", fn, E, moe::kMaxE);
    if (k < 1 || k > moe::kMaxK) return fail(MOE_EINVAL, "%s: k=%d must be in [1, %d]", fn, k, moe::kMaxK);
    if ((long long)T * k > 65536) return fail(MOE_EINVAL, "%s: T*k=%lld exceeds 65536", fn, (long long)T * k);
    CHECK_PTR(idx);
    CHECK_PTR(offsets);
    CHECK_PTR(perm);
    CHECK_OPT_PTR(inv);
    CHECK_OPT_PTR(active);
    if (T == 0) return MOE_OK;
    cudaError_t e = moe::launch_bucket(idx, T * k, E, offsets, perm, inv, active, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_expert_ffn(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *idx, const float *wts,
                   const int32_t *offsets, const int32_t *perm, const int32_t *active, int with_shared, float *m_out,
                   void *ws, size_t ws_bytes, const moe_opts *opts, void *stream) {
    const char *fn = "moe_expert_ffn";
    g_err.clear();
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if ((long long)T * w->k > 65536) return fail(MOE_EINVAL, "%s: T*k exceeds 65536", fn);
    if (int rc = check_expert_ptrs(fn, w, with_shared)) return rc;
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(xe);
    CHECK_PTR(idx);
    CHECK_PTR(wts);
    CHECK_PTR(offsets);
    CHECK_PTR(perm);
    CHECK_PTR(active);
    CHECK_PTR(m_out);
    if (T == 0) return MOE_OK;
    if (int rc = check_ws(fn, w, T, ws, ws_bytes)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(w, T);
    cudaError_t e = run_experts(w, xe, T, offsets, perm, active, with_shared, ws, L, o, st);
    if (e == cudaSuccess)
        e = moe::launch_combine(at<float>(ws, L.y), at<float>(ws, L.sh), wts, T, w->H, w->k, with_shared, nullptr,
                                m_out, nullptr, 0, 1.0f, 0.0f, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_layer_forward(const moe_layer_w *w, const uint16_t *h_in, uint16_t *h_out, int T, void *ws, size_t ws_bytes,
                      const moe_opts *opts, void *stream) {
    const char *fn = "moe_layer_forward";
    g_err.clear();
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if ((long long)T * w->k > 65536) return fail(MOE_EINVAL, "%s: T*k exceeds 65536", fn);
    if (int rc = check_router_ptrs(fn, w)) return rc;
    if (int rc = check_expert_ptrs(fn, w, 1)) return rc;
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(h_in);
    CHECK_PTR(h_out);
    if (T > 0) {
        const char *a = reinterpret_cast<const char *>(h_in), *b = reinterpret_cast<const char *>(h_out);
        const size_t n = sizeof(uint16_t) * (size_t)T * w->H;
        if (a < b + n && b < a + n) return fail(MOE_EINVAL, "%s: h_out overlaps h_in", fn);
    }
    if (T == 0) return MOE_OK;
    if (int rc = check_ws(fn, w, T, ws, ws_bytes)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(w, T);
    double *logits = at<double>(ws, L.logits);
    int32_t *idx = at<int32_t>(ws, L.idx);
    float *wts = at<float>(ws, L.wts);
    uint16_t *xe = at<uint16_t>(ws, L.xe);
    int32_t *offsets = at<int32_t>(ws, L.offsets), *perm = at<int32_t>(ws, L.perm), *inv = at<int32_t>(ws, L.inv);
    int32_t *active = at<int32_t>(ws, L.active);
    cudaError_t e = moe::launch_router_logits(w, h_in, T, o.eps, logits, xe, st);
    if (e == cudaSuccess) e = moe::launch_router_topk(logits, T, w->E, w->k, w->per_expert_scale, idx, wts, st);
    if (e == cudaSuccess) e = moe::launch_bucket(idx, T * w->k, w->E, offsets, perm, inv, active, st);
    if (e == cudaSuccess) e = run_experts(w, xe, T, offsets, perm, active, 1, ws, L, o, st);
    if (e == cudaSuccess)
        e = moe::launch_combine(at<float>(ws, L.y), at<float>(ws, L.sh), wts, T, w->H, w->k, 1, h_in, nullptr, h_out, o.post_norm, o.layer_scalar,
                                o.eps, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_layer_partial(const moe_layer_w *w, const uint16_t *h_in, int T, int e_lo, int e_hi, int with_shared,
                      float *m_out, void *ws, size_t ws_bytes, const moe_opts *opts, void *stream) {
    const char *fn = "moe_layer_partial";
    g_err.clear();
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if ((long long)T * w->k > 65536) return fail(MOE_EINVAL, "%s: T*k exceeds 65536", fn);
    if (e_lo < 0 || e_hi > w->E || e_lo > e_hi)
        return fail(MOE_EINVAL, "%s: expert range [%d, %d) outside [0, %d]", fn, e_lo, e_hi, w->E);
    if (int rc = check_router_ptrs(fn, w)) return rc;
    if (int rc = check_expert_ptrs(fn, w, with_shared)) return rc;
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(h_in);
    CHECK_PTR(m_out);
    if (T == 0) return MOE_OK;
    if (int rc = check_ws(fn, w, T, ws, ws_bytes)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(w, T);
    double *logits = at<double>(ws, L.logits);
    int32_t *idx = at<int32_t>(ws, L.idx);
    float *wts = at<float>(ws, L.wts), *wts_ep = at<float>(ws, L.wts_ep);
    uint16_t *xe = at<uint16_t>(ws, L.xe);
    int32_t *offsets = at<int32_t>(ws, L.offsets), *perm = at<int32_t>(ws, L.perm), *inv = at<int32_t>(ws, L.inv);
    int32_t *active = at<int32_t>(ws, L.active), *active_ep = at<int32_t>(ws, L.active_ep);
    cudaError_t e = moe::launch_router_logits(w, h_in, T, o.eps, logits, xe, st);
    if (e == cudaSuccess) e = moe::launch_router_topk(logits, T, w->E, w->k, w->per_expert_scale, idx, wts, st);
    if (e == cudaSuccess) e = moe::launch_bucket(idx, T * w->k, w->E, offsets, perm, inv, active, st);
    if (e == cudaSuccess) e = moe::launch_ep_select(idx, wts, active, T * w->k, e_lo, e_hi, wts_ep, active_ep, st);
    if (e == cudaSuccess) e = run_experts(w, xe, T, offsets, perm, active_ep, with_shared, ws, L, o, st);
    if (e == cudaSuccess)
        e = moe::launch_combine(at<float>(ws, L.y), at<float>(ws, L.sh), wts_ep, T, w->H, w->k, with_shared, nullptr,
                                m_out, nullptr, 0, 1.0f, o.eps, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_expert_cache_reset(const moe_expert_cache *c, int E, void *stream) {
    const char *fn = "moe_expert_cache_reset";
    g_err.clear();
    if (!c) return fail(MOE_EINVAL, "%s: cache is NULL", fn);
    if (E < 1 || c->slots < 1) return fail(MOE_EINVAL, "%s: E=%d, slots=%d", fn, E, c->slots);
    CHECK_PTR(c->slot_of);
    CHECK_PTR(c->expert_of);
    CHECK_PTR(c->uses);
    CHECK_PTR(c->last);
    CHECK_PTR(c->ctl);
    cudaError_t e = moe::launch_cache_reset(E, c->slots, c->slot_of, c->expert_of, c->uses, c->last, c->ctl,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_layer_forward_cached(const moe_layer_w *w, const moe_expert_cache *c, const uint16_t *h_in, uint16_t *h_out,
                             int T, void *ws, size_t ws_bytes, const moe_opts *opts, void *stream) {
    const char *fn = "moe_layer_forward_cached";
    g_err.clear();
    if (!c) return fail(MOE_EINVAL, "%s: cache is NULL", fn);
    if (int rc = check_dims(fn, w)) return rc;
    if (int rc = check_T(fn, T)) return rc;
    if ((long long)T * w->k > 65536) return fail(MOE_EINVAL, "%s: T*k exceeds 65536", fn);
    const long long need = (long long)T * w->k < w->E ? (long long)T * w->k : w->E;
    if (c->slots < need || c->slots > w->E)
        return fail(MOE_EINVAL, "%s: slots=%d must be in [min(E, T*k)=%lld, E=%d]", fn, c->slots, need, w->E);
    if (int rc = check_router_ptrs(fn, w)) return rc;
    // the shared expert is resident; the routed experts come from the cache
    moe_layer_w wc = *w;
    wc.E = c->slots;
    wc.gate = c->gate;
    wc.up = c->up;
    wc.down = c->down;
    if (int rc = check_expert_ptrs(fn, &wc, 1)) return rc;
    CHECK_PTR(c->pool_gate.q);
    CHECK_PTR(c->pool_gate.sb);
    CHECK_PTR(c->pool_up.q);
    CHECK_PTR(c->pool_up.sb);
    CHECK_PTR(c->pool_down.q);
    CHECK_PTR(c->pool_down.sb);
    CHECK_PTR(c->slot_of);
    CHECK_PTR(c->expert_of);
    CHECK_PTR(c->uses);
    CHECK_PTR(c->last);
    CHECK_PTR(c->ctl);
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(h_in);
    CHECK_PTR(h_out);
    if (T == 0) return MOE_OK;
    if (int rc = check_ws(fn, w, T, ws, ws_bytes)) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(w, T);
    double *logits = at<double>(ws, L.logits);
    int32_t *idx = at<int32_t>(ws, L.idx), *idx_c = at<int32_t>(ws, L.idx_c), *miss = at<int32_t>(ws, L.miss);
    float *wts = at<float>(ws, L.wts);
    uint16_t *xe = at<uint16_t>(ws, L.xe);
    int32_t *offsets = at<int32_t>(ws, L.offsets), *perm = at<int32_t>(ws, L.perm), *inv = at<int32_t>(ws, L.inv);
    int32_t *active = at<int32_t>(ws, L.active);
    const moe_qmat pool[3] = {c->pool_gate, c->pool_up, c->pool_down}, cache[3] = {c->gate, c->up, c->down};
    cudaError_t e = moe::launch_router_logits(w, h_in, T, o.eps, logits, xe, st);
    if (e == cudaSuccess) e = moe::launch_router_topk(logits, T, w->E, w->k, w->per_expert_scale, idx, wts, st);
    if (e == cudaSuccess)
        e = moe::launch_residency(idx, T * w->k, w->E, c->slots, c->slot_of, c->expert_of, c->uses, c->last, c->ctl,
                                  miss, idx_c, st);
    if (e == cudaSuccess) e = moe::launch_fill(w, pool, cache, miss, st);
    if (e == cudaSuccess) e = moe::launch_bucket(idx_c, T * w->k, c->slots, offsets, perm, inv, active, st);
    if (e == cudaSuccess) e = run_experts(&wc, xe, T, offsets, perm, active, 1, ws, L, o, st);
    if (e == cudaSuccess)
        e = moe::launch_combine(at<float>(ws, L.y), at<float>(ws, L.sh), wts, T, w->H, w->k, 1, h_in, nullptr, h_out,
                                o.post_norm, o.layer_scalar, o.eps, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_combine(const uint16_t *h_in, const float *m, uint16_t *h_out, int T, int H, const moe_opts *opts,
                void *stream) {
    const char *fn = "moe_combine";
    g_err.clear();
    if (H < 64 || H % 64 || H > 8192) return fail(MOE_EINVAL, "%s: H=%d must be a multiple of 64 in [64, 8192]", fn, H);
    if (int rc = check_T(fn, T)) return rc;
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(h_in);
    CHECK_PTR(m);
    CHECK_PTR(h_out);
    if (T == 0) return MOE_OK;
    cudaError_t e = moe::launch_combine(nullptr, m, nullptr, T, H, 0, 1, h_in, nullptr, h_out, o.post_norm,
                                        o.layer_scalar, o.eps, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

size_t moe_decode_stack_workspace_size(const moe_layer_w *w, int T) {
    if (check_dims("moe_decode_stack_workspace_size", w) || T < 1 || T > moe::decode_stack_max_tokens()) return 0;
    return moe::decode_stack_ws_bytes(w, T);
}

// Grid of the persistent decode kernel on `dev` (one CTA per SM), cached.
static cudaError_t decode_grid_of(int dev, int *grid) {
    static std::mutex mu;
    static int grids[64] = {0};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (grids[dev] == 0) {
        int coop = 0;
        cudaError_t e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        if (e != cudaSuccess) return e;
        if (!coop) {
            grids[dev] = -1;
        } else {
            e = moe::decode_stack_grid(dev, &grids[dev]);
            if (e != cudaSuccess) return e;
            if (grids[dev] <= 0) grids[dev] = -1;
        }
    }
    *grid = grids[dev];
    return cudaSuccess;
}

int moe_decode_stack_fits(const moe_layer_w *w, int T, void *stream) {
    g_err.clear();
    if (!w || check_dims("moe_decode_stack_fits", w) || T < 1 || T > moe::decode_stack_max_tokens()) return 0;
    if (w->H > 4096 || T * w->H > moe::decode_stack_stage_floats()) return 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0, grid = 0;
    if ((st ? cudaStreamGetDevice(st, &dev) : cudaGetDevice(&dev)) != cudaSuccess) return 0;
    if (decode_grid_of(dev, &grid) != cudaSuccess || grid <= 0) return 0;
    return moe::decode_stack_fits(w, T, grid, 0) ? 1 : 0;
}

int moe_decode_stack(const moe_layer_w *layers, int L, const uint16_t *h_in, int chained, uint16_t *h_out, int T,
                     void *ws, size_t ws_bytes, const moe_opts *opts, void *stream) {
    const char *fn = "moe_decode_stack";
    g_err.clear();
    if (!layers) return fail(MOE_EINVAL, "%s: layers is NULL", fn);
    if (L < 1 || L > moe::decode_stack_max_layers())
        return fail(MOE_EINVAL, "%s: L=%d must be in [1, %d]", fn, L, moe::decode_stack_max_layers());
    if (T < 0 || T > moe::decode_stack_max_tokens())
        return fail(MOE_EINVAL, "%s: T=%d must be in [0, %d]", fn, T, moe::decode_stack_max_tokens());
    const moe_layer_w &w0 = layers[0];
    for (int l = 0; l < L; ++l) {
        const moe_layer_w *w = &layers[l];
        if (int rc = check_dims(fn, w)) return rc;
        if (w->H != w0.H || w->E != w0.E || w->k != w0.k || w->I != w0.I || w->Is != w0.Is)
            return fail(MOE_EINVAL, "%s: layer %d has a different shape from layer 0", fn, l);
        if (int rc = check_router_ptrs(fn, w)) return rc;
        if (int rc = check_expert_ptrs(fn, w, 1)) return rc;
    }
    if (w0.H > 4096) return fail(MOE_EINVAL, "%s: H=%d exceeds 4096", fn, w0.H);
    if (T * w0.H > moe::decode_stack_stage_floats())
        return fail(MOE_EINVAL, "%s: T*H=%d exceeds %d", fn, T * w0.H, moe::decode_stack_stage_floats());
    const moe_opts o = resolve_opts(opts);
    if (int rc = check_opts(fn, o)) return rc;
    CHECK_PTR(h_in);
    CHECK_PTR(h_out);
    if (T == 0) return MOE_OK;
    const size_t need = moe::decode_stack_ws_bytes(&w0, T);
    if (!ws) return fail(MOE_EWORKSPACE, "%s: workspace is NULL (need %zu bytes)", fn, need);
    if (!aligned16(ws)) return fail(MOE_EALIGN, "%s: workspace is not 16-byte aligned", fn);
    if (ws_bytes < need) return fail(MOE_EWORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn, ws_bytes, need);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    cudaError_t e = st ? cudaStreamGetDevice(st, &dev) : cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    if (dev < 0 || dev >= 64) return fail(MOE_EINVAL, "%s: device %d out of range", fn, dev);
    int grid = 0;
    if ((e = decode_grid_of(dev, &grid)) != cudaSuccess) return cuda_fail(e, fn);
    if (grid <= 0)
        return fail(MOE_EINVAL, "%s: device %d cannot run the decode kernel (cooperative launch, one CTA per SM)", fn,
                    dev);
    if (!moe::decode_stack_fits(&w0, T, grid, o.force_path))
        return fail(MOE_EINVAL, "%s: T=%d with H=%d, E=%d does not fit the kernel's shared memory", fn, T, w0.H, w0.E);
    e = moe::launch_decode_stack(layers, L, h_in, chained, h_out, T, ws, o, grid, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

size_t moe_qmat_gemv_workspace_size(void) { return 256; }

int moe_qmat_gemv(const moe_qmat *w, int rows, int cols, const uint16_t *x, int T, float *y, void *ws,
                  size_t ws_bytes, void *stream) {
    const char *fn = "moe_qmat_gemv";
    g_err.clear();
    if (!w) return fail(MOE_EINVAL, "%s: matrix is NULL", fn);
    if (rows < 32 || rows % 32) return fail(MOE_EINVAL, "%s: rows=%d must be a positive multiple of 32", fn, rows);
    if (cols < 64 || cols % 64 || cols > kMaxDim)
        return fail(MOE_EINVAL, "%s: cols=%d must be a multiple of 64 in [64, %d]", fn, cols, kMaxDim);
    if (T < 1 || T > 8) return fail(MOE_EINVAL, "%s: T=%d must be in [1, 8]", fn, T);
    if (moe::qmat_gemv_smem(cols, T) > (size_t)200 * 1024)
        return fail(MOE_EINVAL, "%s: T=%d rows of %d columns do not fit the shared-memory stage", fn, T, cols);
    CHECK_PTR(w->q);
    CHECK_PTR(w->sb);
    CHECK_PTR(x);
    CHECK_PTR(y);
    CHECK_PTR(ws);
    if (ws_bytes < moe_qmat_gemv_workspace_size())
        return fail(MOE_EWORKSPACE, "%s: workspace of %zu bytes, need %zu", fn, ws_bytes, moe_qmat_gemv_workspace_size());
    cudaError_t e = moe::launch_qmat_gemv(*w, rows, cols, x, T, y, static_cast<unsigned *>(ws),
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, fn);
}

int moe_workspace_status(const void *ws) {
    const char *fn = "moe_workspace_status";
    g_err.clear();
    if (!ws) return fail(MOE_EINVAL, "%s: workspace is NULL", fn);
    int code[2] = {0, 0};
    cudaError_t e = cudaMemcpy(code, static_cast<const char *>(ws) + kStatusOffset, sizeof code, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    if (code[0] != 0) {
        static const char *what[] = {"", "wait for weights timed out", "wait for a free weight slot timed out",
                                     "wait for a weight tile timed out", "wait for a free weight tile timed out",
                                     "wait for a token tile timed out", "wait for a free token tile timed out",
                                     "wait for the accumulator timed out", "wait for the epilogue timed out"};
        return fail(MOE_EDEVICE, "%s: device error %d (%s)", fn, code[0],
                    (code[0] > 0 && code[0] < 9) ? what[code[0]] : "?");
    }
    if (code[1] != 0)
        return fail(MOE_EDEVICE, "%s: %s outside the FP16 range of the tensor-core path; outputs are invalid "
                    "(%s)", fn, code[1] == 1 ? "a weight s*q + b" : "a SwiGLU value silu(g)*u",
                    code[1] == 1 ? "force_path 1 or 3 computes this layer" : "force_path 1 computes this layer");
    return MOE_OK;
}

int moe_decode_stack_status(const void *ws) {
    const char *fn = "moe_decode_stack_status";
    g_err.clear();
    if (!ws) return fail(MOE_EINVAL, "%s: workspace is NULL", fn);
    int code = 0;
    cudaError_t e = cudaMemcpy(&code, static_cast<const char *>(ws) + moe::decode_stack_status_offset(), sizeof code,
                               cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    if (code != 0) {
        static const char *what[] = {"", "grid barrier timed out", "wait for weights timed out",
                                     "wait for a free ring slot timed out",
                                     "wait for another CTA's gate/up units timed out",
                                     "wait for a ring slot's hand-over timed out",
                                     "wait for the routing tables timed out",
                                     "wait for a staged down-projection input timed out",
                                     "wait for another CTA's router logits timed out"};
        return fail(MOE_EDEVICE, "%s: device error %d (%s)", fn, code, (code > 0 && code < 9) ? what[code] : "?");
    }
    return MOE_OK;
}

}  // extern "C"
