// GOLD key compression and TokenCat decompression (csrc/gold.cu): the two matrix products
// run as cuBLASLt GEMMs (bf16 operands, fp32 accumulation); RMSNorm is a kernel of ours.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace goldwkv {

// c [N][Dc] = x [N][D] . w_kd^T, w_kd [Dc][D]; bf16, fp32 accumulation.  false on failure.
bool gold_gemm_compress(const void* x, const void* w_kd, void* c, long N, int D, int Dc,
                        void* lt_workspace, size_t lt_bytes, cudaStream_t st);

// z [N][D] fp32 = concat(x0 [N][D], c [N][Dc]) . w_ku^T, w_ku [D][D + Dc] bf16: the
// concatenation is written to cat [N][D + Dc] (bf16 scratch), then one GEMM.  false on
// failure.
bool gold_gemm_decompress(const void* x0, const void* c, const void* w_ku, void* cat, float* z,
                          long N, int D, int Dc, void* lt_workspace, size_t lt_bytes,
                          cudaStream_t st);

// out [N][D] bf16 = z / sqrt(mean(z^2) + eps) * gamma (gamma null = 1), per row.
cudaError_t launch_rmsnorm_rows(const float* z, const float* gamma, float eps, void* out, long N,
                                int D, cudaStream_t st);

}  // namespace goldwkv
