// Kernel launchers behind the libgoldwkv C ABI (not exported).
#pragma once

#include <cuda.h>
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

// ---- chunked tensor-core prefill (bf16 I/O)
// TMA descriptor of a [B][T][H][64] bf16 tensor: box 64 channels x 1 head x 64 tokens.
bool make_token_map(CUtensorMap* m, const void* base, int B, int T, int H);

// Fast path (one-sided decay factorisation, warp-specialised pipeline).  maps: r, k, v,
// omega, y.  For each (b,h) it writes y and the final state, or stops at the first chunk
// whose decay range it cannot take and records that chunk in handoff_chunk[bh] (-1: done)
// with the state entering it in handoff_state[bh].  y_raw != nullptr: fp32 y rows there.
cudaError_t launch_chunked_fast(const CUtensorMap* maps, const float* u, const float* s_in,
                                float* s_out, void* y, float* y_raw, int B, int T, int H, int* status,
                                int* handoff_chunk, float* handoff_state, long long budget,
                                cudaStream_t st);

// Level-factorised path (any decay).  start_chunk == nullptr: every (b,h) from chunk 0 with
// state s_in; otherwise (b,h) resumes at start_chunk[bh] (skipped if < 0) from
// handoff_state.  status: device word set to 1 if a bounded wait expired.
cudaError_t launch_chunked_levels(const CUtensorMap* maps, const float* u, const float* s_in,
                                  float* s_out, float* y_raw, int B, int T, int H, int* status,
                                  const int* start_chunk, const float* handoff_state,
                                  long long spin_budget, cudaStream_t st);
size_t chunked_smem_bytes();
size_t fast_smem_bytes();

}  // namespace goldwkv
