// noalloc.cu -- coli_moe_layer_noalloc: the whole layer with its scratch in a static device array.
//
// Some callers cannot give the library a workspace: a plugin inside a serving engine whose GPU
// memory pool is fixed when the engine starts, or a real-time loop that must never pay for
// cudaMalloc's device-wide synchronisation.  They still own their input and output buffers, so
// this entry point takes those, and keeps everything else it needs in one file-scope
// `__device__` array of COLI_MOE_STATIC_SCRATCH_BYTES bytes.  Every GPU that loads the library
// holds that array until the process exits.
//
// The array's name, in host code, is only a host-side handle for the symbol, not a device
// address; the device address is obtained once per device with cudaGetSymbolAddress (with that
// device current) and cached.  That set-up happens inside the first call on each device.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "coli_moe.h"
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_static_scratch[COLI_MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_static_scratch on the current device (set up once per device).
coli_status static_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COLI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return COLI_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return COLI_OK;
}

}  // namespace

extern "C" coli_status coli_moe_layer_noalloc(const coli_moe_config *cfg, const coli_moe_weights *w,
                                              const void *x, int T, float *out,
                                              int32_t *topk_ids_out, float *topk_w_out,
                                              void *stream) {
    coli_status s = coli_moe_check_config(cfg);
    if (s != COLI_OK) return s;
    if (T < 0) return COLI_ERR_SHAPE;
    if (T == 0) return COLI_OK;
    size_t need = 0;
    s = coli_moe_workspace_size(cfg, T, &need);
    if (s != COLI_OK) return s;
    if (need > static_cast<size_t>(COLI_MOE_STATIC_SCRATCH_BYTES)) return COLI_ERR_WORKSPACE;
    // every argument check before the first GPU operation: a rejected call launches nothing
    s = coli::layer_args_status(cfg, w, x, T, out, topk_ids_out, topk_w_out);
    if (s != COLI_OK) return s;
    void *ws = nullptr;
    s = static_scratch(&ws);
    if (s != COLI_OK) return s;
    // The array keeps the previous call's contents: the header (error word and counters) must
    // start at zero for every call.
    if (cudaMemsetAsync(ws, 0, coli::WS_HEADER, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return COLI_ERR_CUDA;
    return coli_moe_layer(cfg, w, x, T, out, topk_ids_out, topk_w_out, ws,
                          static_cast<size_t>(COLI_MOE_STATIC_SCRATCH_BYTES), stream);
}

extern "C" coli_status coli_moe_noalloc_error_word(void *stream, int *code) {
    if (!code) return COLI_ERR_INVALID_ARG;
    void *ws = nullptr;
    const coli_status s = static_scratch(&ws);
    if (s != COLI_OK) return s;
    return coli_moe_error_word(ws, stream, code);
}
