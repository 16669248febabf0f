// moe_internal.h -- launchers shared between the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe_api.h"

namespace moe {

// Record `msg` as this host thread's moe_last_error() text; returns `code`.
int set_last_error(int code, const char *msg);

// The device that runs launches on `st`: the stream's own (NULL: the current
// device).  While `st` is being captured into a CUDA graph the current device
// is taken instead (the captured launches run there): asking a capturing
// stream for its device ended the capture on the warp-MMA path, and the
// capture-status query is the one stream query a capture allows.
inline cudaError_t stream_device(cudaStream_t st, int *dev) {
    if (st) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        const cudaError_t e = cudaStreamIsCapturing(st, &cs);
        if (e != cudaSuccess) return e;
        if (cs == cudaStreamCaptureStatusNone) return cudaStreamGetDevice(st, dev);
    }
    return cudaGetDevice(dev);
}

// Raise a kernel's dynamic shared memory limit once (per process) to at
// least `bytes`.  A no-op below 48 KiB.
cudaError_t ensure_smem(const void *kernel, size_t bytes);

size_t router_logits_smem(int H);
cudaError_t launch_router_logits(const moe_layer_w *w, const uint16_t *h, int T, float eps, double *logits,
                                 uint16_t *xe, cudaStream_t st);
cudaError_t launch_router_topk(const double *logits, int T, int E, int k, const uint16_t *pes, int32_t *idx,
                               float *wts, cudaStream_t st);
cudaError_t launch_bucket(const int32_t *idx, int n_pairs, int E, int32_t *offsets, int32_t *perm, int32_t *inv,
                          int32_t *active, cudaStream_t st);
cudaError_t launch_prepare_qmat(const uint32_t *q, const uint16_t *s, const uint16_t *b, int n_mat, int rows,
                                int cols, uint32_t *q_out, uint32_t *sb_out, cudaStream_t st);

// Intermediate buffers of the expert part (all device, from the workspace).
struct FfnBuffers {
    float *a_routed;  // [T*k, I]  SwiGLU output, by bucketed position
    float *a_shared;  // [T, Is]
    float *y;         // [T*k, H]  routed expert outputs, by pair id t*k+s
    float *sh;        // [T, H]    shared expert output
};

size_t gemv_smem_bytes(int cols, int nt);
cudaError_t launch_expert_gemv(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                               const int32_t *perm, const int32_t *active, int with_shared, const FfnBuffers &b,
                               cudaStream_t st);
// One tiled 4-bit matrix times up to 8 bf16 rows (moe_gemv.cu); ctr: a device word (reset by the launch).
size_t qmat_gemv_smem(int cols, int T);
cudaError_t launch_qmat_gemv(const moe_qmat &w, int rows, int cols, const uint16_t *x, int T, float *y,
                             unsigned *ctr, cudaStream_t st);
// Tensor-core grouped GEMM path (moe_mma.cu).
struct MmaBuffers {
    uint16_t *xg;   // [T + T*k, H]    FP16 token rows (shared, then bucketed pairs), chunk-permuted
    uint16_t *act;  // [T + T*k, Kmax] FP16 SwiGLU rows, chunk-permuted, Kmax = max(I, Is)
    float *y;       // [T*k, H]  routed expert outputs, by pair id t*k+s
    float *sh;      // [T, H]    shared expert output
    int *err;       // device error word (0 = ok): a bounded wait ran out
    int *range_err; // device word (0 = ok): a weight or SwiGLU value outside the FP16 range
};
size_t mma_xg_bytes(const moe_layer_w *w, int T);
// FP16 token rows for the tensor-core paths: row r < T token r, row T + j the token of bucketed pair j.
// odd_div16: the odd input columns (stored places 2, 3, 6, 7 of every 8) hold x / 16, rounded once
// (the warp-MMA path's operand encoding); otherwise every value is x.
cudaError_t launch_gather_tokens(const uint16_t *xe, const int32_t *perm, int T, int k, int H, uint16_t *xg,
                                 cudaStream_t st, bool odd_div16 = false);
// Weight-stationary warp-MMA expert FFN (moe_wsmma.cu): same buffers as launch_expert_mma.
bool wsmma_supported(const moe_layer_w *w);
cudaError_t launch_expert_wsmma(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                                const int32_t *perm, const int32_t *active, int with_shared, const MmaBuffers &b,
                                cudaStream_t st);
size_t mma_act_bytes(const moe_layer_w *w, int T);
cudaError_t launch_expert_mma(const moe_layer_w *w, const uint16_t *xe, int T, const int32_t *offsets,
                              const int32_t *perm, const int32_t *active, int with_shared, const MmaBuffers &b,
                              cudaStream_t st);

// mode 0: m_out[t] = sum_s w y + sh ; mode 1: h_out = bf16((h + rmsnorm(m)) * scalar) (or no norm)
cudaError_t launch_combine(const float *y, const float *sh, const float *wts, int T, int H, int k, int with_shared,
                           const uint16_t *h_in, float *m_out, uint16_t *h_out, int post_norm, float layer_scalar,
                           float eps, cudaStream_t st);

// Expert-parallel selection: gate weights of pairs outside [e_lo, e_hi) set to 0, active list filtered.
cudaError_t launch_ep_select(const int32_t *idx, const float *wts, const int32_t *active, int n, int e_lo, int e_hi,
                             float *wts_out, int32_t *active_out, cudaStream_t st);

// Tiered expert residency (moe_cache.cu).
cudaError_t launch_residency(const int32_t *idx, int n, int E, int C, int32_t *slot_of, int32_t *expert_of,
                             uint32_t *uses, uint32_t *last, uint32_t *ctl, int32_t *miss, int32_t *idx_c,
                             cudaStream_t st);
cudaError_t launch_fill(const moe_layer_w *w, const moe_qmat pool[3], const moe_qmat cache[3], const int32_t *miss,
                        cudaStream_t st);
cudaError_t launch_cache_reset(int E, int C, int32_t *slot_of, int32_t *expert_of, uint32_t *uses, uint32_t *last,
                               uint32_t *ctl, cudaStream_t st);

// Persistent decode kernel over a stack of layers (moe_decode.cu).
size_t decode_stack_smem();
size_t decode_stack_ws_bytes(const moe_layer_w *w, int T);
size_t decode_stack_status_offset();
int decode_stack_max_tokens();
bool decode_stack_fits(const moe_layer_w *w, int T, int grid, int force_path);
int decode_stack_max_layers();
int decode_stack_stage_floats();
cudaError_t decode_stack_grid(int device, int *grid);
cudaError_t launch_decode_stack(const moe_layer_w *layers, int L, const uint16_t *h_in, int chained,
                                uint16_t *h_out, int T, void *ws, const moe_opts &o, int grid, cudaStream_t st);

}  // namespace moe
