// Allocation-free prefill: wkv6_prefill with its workspace taken from a scratch array
// compiled into the library instead of from the caller.  Contract in include/goldwkv.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "goldwkv.h"

namespace {

// One scratch per device, zero when the library's device code is loaded.  Its first word is
// the chunked path's status word: the kernels only ever set it (when a bounded wait
// expires), nothing reads it on this path, so its value never changes a result.
static __device__ __align__(256) uint8_t g_prefill_scratch[WKV6_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch, looked up once per device (with that device
// current) and cached; nullptr if the lookup fails.
void* scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" wkv_status wkv6_prefill_static(const void* r, const void* k, const void* v,
                                          const void* omega, const float* u,
                                          const float* state_in, float* state_out, void* y,
                                          int B, int T, int H, int D, wkv_dtype io,
                                          const wkv_ln* ln, void* stream) {
    if (B < 0 || T < 0 || H < 0 || (io != WKV_F32 && io != WKV_BF16)) return WKV_ERR_INVALID_ARG;
    size_t need = 0;
    if (B > 0 && T > 0 && H > 0)
        need = wkv6_prefill_workspace_bytes(B, T, H, D, io, ln != nullptr, WKV_ALGO_AUTO);
    if (need > WKV6_STATIC_SCRATCH_BYTES) return WKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = scratch_for_current_device();
        if (scratch == nullptr) return WKV_ERR_CUDA;
    }
    return wkv6_prefill(r, k, v, omega, u, state_in, state_out, y, B, T, H, D, io, ln, scratch,
                        need > 0 ? (size_t)WKV6_STATIC_SCRATCH_BYTES : 0, stream);
}
