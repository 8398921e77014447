// Device helpers shared by the libgoldwkv kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace goldwkv {

constexpr int kHeadSize = 64;   // D: the only head size the kernels are built for

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Decay factor of one channel: w = exp(-exp(omega)), in (0, 1].  Accurate libm exp on
// both steps; the kernels that call this are bound by memory or by the serial recurrence.
__device__ __forceinline__ float decay_from_logit(float omega) {
    return expf(-expf(omega));
}

// Debug builds (-DGW_DEBUG, built as libgoldwkv_debug.so): device-side checks of the
// indices a copy or a store is about to use.  A failed check sets bit 1 of the kernel's
// status word (*status |= 2) and the guarded access is skipped; nothing traps.  In release
// builds the check is the constant true and costs nothing.
#ifdef GW_DEBUG
__device__ __forceinline__ bool gw_check(int* status, bool ok) {
    if (!ok) atomicOr(status, 2);
    return ok;
}
#else
__device__ __forceinline__ constexpr bool gw_check(int*, bool) { return true; }
#endif

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace goldwkv
