// moe_noalloc.cu -- moe_layer_forward for callers that cannot allocate device
// memory (see moe_layer_forward_noalloc in include/moe_api.h).
//
// The scratch that moe_layer_forward takes as a caller-provided workspace
// lives here in one file-scope __device__ array instead.  Host code never
// uses the array's name as an address (on the host it only names a stand-in
// object); the device address is looked up with cudaGetSymbolAddress once per
// device, with that device current, and then handed to moe_layer_forward.
#include <cstdio>
#include <mutex>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev`, looked up once per device
// with that device current (the previous current device is restored).
int scratch_on(int dev, void **out) {
    if (dev < 0 || dev >= kMaxDevices) return moe::set_last_error(MOE_EINVAL, "moe_layer_forward_noalloc: device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        int prev = -1;
        cudaError_t e = cudaGetDevice(&prev);
        if (e == cudaSuccess && prev != dev) e = cudaSetDevice(dev);
        void *p = nullptr;
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (prev >= 0 && prev != dev) cudaSetDevice(prev);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "moe_layer_forward_noalloc: cudaGetSymbolAddress failed on device %d: %s", dev,
                     cudaGetErrorString(e));
            return moe::set_last_error(MOE_ECUDA, msg);
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

int moe_layer_forward_noalloc(const moe_layer_w *w, const uint16_t *h_in, uint16_t *h_out, int T,
                              const moe_opts *opts, void *stream) {
    if (T == 0 || !w) return moe_layer_forward(w, h_in, h_out, T, nullptr, 0, opts, stream);
    const size_t need = moe_workspace_size(w, T);
    if (need == 0) return moe_layer_forward(w, h_in, h_out, T, nullptr, 0, opts, stream);  // reports the bad size
    if (need > kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "moe_layer_forward_noalloc: T=%d needs %zu bytes of scratch but the static scratch holds %zu; "
                 "use moe_layer_forward with a caller-provided workspace",
                 T, need, kStaticScratchBytes);
        return moe::set_last_error(MOE_EWORKSPACE, msg);
    }
    int dev = 0;
    cudaError_t e = stream ? cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &dev) : cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "moe_layer_forward_noalloc: cannot tell the stream's device: %s", cudaGetErrorString(e));
        return moe::set_last_error(MOE_ECUDA, msg);
    }
    void *scratch = nullptr;
    if (int rc = scratch_on(dev, &scratch)) return rc;
    return moe_layer_forward(w, h_in, h_out, T, scratch, kStaticScratchBytes, opts, stream);
}

int moe_noalloc_status(void *stream) {
    int dev = 0;
    cudaError_t e = stream ? cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &dev) : cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "moe_noalloc_status: cannot tell the stream's device: %s", cudaGetErrorString(e));
        return moe::set_last_error(MOE_ECUDA, msg);
    }
    void *scratch = nullptr;
    if (int rc = scratch_on(dev, &scratch)) return rc;
    if (stream && (e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "moe_noalloc_status: %s", cudaGetErrorString(e));
        return moe::set_last_error(MOE_ECUDA, msg);
    }
    return moe_workspace_status(scratch);
}

}  // extern "C"
