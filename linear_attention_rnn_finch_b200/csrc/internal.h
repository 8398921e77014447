// Kernel launchers behind the libgoldwkv C ABI (not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace goldwkv {

// Token-by-token recurrence (fp32 math).  y_raw != nullptr: write fp32 un-normalised y
// there instead of y.
cudaError_t launch_recurrent(const void* r, const void* k, const void* v, const void* omega,
                             const float* u, const float* s_in, float* s_out, void* y,
                             float* y_raw, int B, int T, int H, bool bf16, cudaStream_t st);

// One decode step, state in place.  y_raw as above.
cudaError_t launch_decode(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, float* state, void* y, float* y_raw, int B, int H,
                          bool bf16, cudaStream_t st);

// LayerNorm of `rows` rows of C fp32 values into `out` (fp32 or bf16); out may equal x.
cudaError_t launch_layernorm_rows(const float* x, const float* gamma, const float* beta,
                                  float eps, void* out, long rows, int C, bool bf16,
                                  cudaStream_t st);

}  // namespace goldwkv
