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

// Chunked tensor-core prefill (bf16 I/O).  y_raw != nullptr: fp32 y rows go there (for a
// LayerNorm pass) instead of bf16 y.  status: device word set to 1 if a bounded wait
// expired.  spin_budget: SM cycles each wait may spin.
cudaError_t launch_chunked(const void* r, const void* k, const void* v, const void* omega,
                           const float* u, const float* s_in, float* s_out, void* y,
                           float* y_raw, int B, int T, int H, int* status, long long spin_budget,
                           cudaStream_t st);
size_t chunked_smem_bytes();

}  // namespace goldwkv
