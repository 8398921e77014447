// Allocation-free prefill: wkv6_prefill with its workspace taken from a scratch array
// compiled into the library instead of from the caller.  Contract in include/goldwkv.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "goldwkv.h"
#include "internal.h"

namespace {

// One scratch per device, zero when the library's device code is loaded.  Its first word is
// the chunked path's status word: a kernel sets it when one of its bounded waits expires, and
// wkv6_prefill_static_status reads and clears it.
static __device__ __align__(256) uint8_t g_prefill_scratch[WKV6_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
struct Cached {
    CUcontext ctx;  // context the address was looked up in
    void* ptr;
};
Cached g_scratch[kMaxDevices] = {};

using CtxGetCurrent = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point query (no libcuda link needed).
CtxGetCurrent ctx_get_current() {
    static CtxGetCurrent fn = []() -> CtxGetCurrent {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetCurrent>(p);
    }();
    return fn;
}

// Device address of this device's scratch in the current context; nullptr if the lookup
// fails.  The address is cached per device together with the context it belongs to and
// looked up again when the current context differs (a device reset makes a new primary
// context, whose module -- and scratch -- are new).
void* scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    // cudaFree(nullptr) makes the device's primary context current if none is yet
    CUcontext ctx = nullptr;
    CtxGetCurrent get = ctx_get_current();
    if (get == nullptr || cudaFree(nullptr) != cudaSuccess || get(&ctx) != CUDA_SUCCESS ||
        ctx == nullptr) {
        (void)cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    Cached& c = g_scratch[dev];
    if (c.ptr == nullptr || c.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        c = Cached{ctx, p};
    }
    return c.ptr;
}

}  // namespace

namespace goldwkv {

CUcontext current_context() {
    CUcontext ctx = nullptr;
    CtxGetCurrent get = ctx_get_current();
    if (get == nullptr || get(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

}  // namespace goldwkv

extern "C" wkv_status wkv6_prefill_static(const void* r, const void* k, const void* v,
                                          const void* omega, const float* u,
                                          const float* state_in, float* state_out, void* y,
                                          int B, int T, int H, int D, wkv_dtype io,
                                          const wkv_ln* ln, void* stream) {
    if (B < 0 || T < 0 || H < 0 || (io != WKV_F32 && io != WKV_BF16)) return WKV_ERR_INVALID_ARG;
    // the sequence split is capped so that the workspace fits the scratch
    const size_t need = goldwkv::prefill_bytes_within(B, T, H, D, io, ln != nullptr,
                                                      WKV6_STATIC_SCRATCH_BYTES);
    if (need > WKV6_STATIC_SCRATCH_BYTES) return WKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = scratch_for_current_device();
        if (scratch == nullptr) return WKV_ERR_CUDA;
    }
    return goldwkv::prefill_within(r, k, v, omega, u, state_in, state_out, y, B, T, H, D, io,
                                   ln, scratch,
                                   need > 0 ? (size_t)WKV6_STATIC_SCRATCH_BYTES : 0, stream);
}

extern "C" wkv_status wkv6_prefill_static_status(void* stream) {
    void* scratch = scratch_for_current_device();
    if (scratch == nullptr) return WKV_ERR_CUDA;
    return wkv6_workspace_status(scratch, stream);
}
