// GOLD key compression and TokenCat decompression: the two matrix products run in
// gold_gemm (csrc/gold_gemm_sm100.cu, tcgen05, bf16 operands, fp32 accumulation), with the
// RMSNorm in its epilogue when a row fits one cluster, else in launch_rmsnorm_rows.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace goldwkv {

// What gold_gemm writes: the product as bf16, as fp32, or RMSNorm-ed over each row's nout
// values (times gamma, null = 1) as bf16.
enum class GoldOut { kBf16, kF32, kRmsNormBf16 };

// C [M][nout] = [a1 | a2] . w^T on tcgen05 (csrc/gold_gemm_sm100.cu): a1 [M][K1] and a2
// [M][K2] bf16 (a2 unused when K2 == 0), w [nout][K1 + K2] bf16, fp32 accumulation; K1,
// K2, nout multiples of 8, pointers 16-byte aligned.  kRmsNormBf16 requires
// gold_rmsnorm_fusable(nout) (a row's column tiles fit one thread-block cluster).  *status
// is set to 1 if a bounded wait expires (results then undefined).
cudaError_t gold_gemm(const void* a1, long K1, const void* a2, long K2, const void* w, long nout,
                      long M, GoldOut out, void* C, const float* gamma, float eps, int* status,
                      long long budget, cudaStream_t st);
bool gold_rmsnorm_fusable(int D);

// out [N][D] bf16 = z / sqrt(mean(z^2) + eps) * gamma (gamma null = 1), per row.
cudaError_t launch_rmsnorm_rows(const float* z, const float* gamma, float eps, void* out, long N,
                                int D, cudaStream_t st);

}  // namespace goldwkv
