// GOLD key compression and TokenCat decompression (GoldFinch review page, section 3.4 "GOLD
// Key Compression and TokenCat Decompression"):
//     c_t   = x_t W_KD                                   (D -> Dc = D/16)
//     k^D_t = RMSNorm(concat(x0_t, c_t) W_KU)            (D + Dc -> D)
// Both products are plain dense GEMMs and run through cuBLASLt on the tensor cores (bf16
// operands, fp32 accumulation).  The concatenation [x0 | c] is copied into the workspace
// by a kernel of ours (16-byte moves) so that the decompression is one GEMM over
// K = D + Dc, its fp32 output written once; RMSNorm over the D outputs of a token is our
// kernel too.
//
// Row-major [rows][cols] matrices are cuBLAS column-major [cols x rows] matrices, so with
// the weights given as the rows of each map (w[out][in]) every product is a "TN" GEMM:
// C^T (out x N) = W (in x out, transposed) . X^T (in x N).
#include <cublasLt.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "gold.h"

namespace goldwkv {

namespace {

// One cuBLASLt handle for the process, created on first use (host state only).
cublasLtHandle_t lt_handle() {
    static std::once_flag once;
    static cublasLtHandle_t h = nullptr;
    std::call_once(once, [] {
        if (cublasLtCreate(&h) != CUBLAS_STATUS_SUCCESS) h = nullptr;
    });
    return h;
}

// D (m x n, ldd, type dtype) = alpha * op_T(A) . B + beta * D, A stored (k x m, lda), B
// (k x n, ldb), both bf16; fp32 compute.
bool gemm_tn(int m, int n, int k, const void* A, int lda, const void* B, int ldb, float beta,
             void* Dm, cudaDataType_t dtype, int ldd, void* ws, size_t ws_bytes, cudaStream_t st) {
    cublasLtHandle_t h = lt_handle();
    if (h == nullptr) return false;
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, ld = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    bool ok = false;
    do {
        if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
            break;
        const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
        if (cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) !=
                CUBLAS_STATUS_SUCCESS ||
            cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)) !=
                CUBLAS_STATUS_SUCCESS)
            break;
        if (cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, k, m, lda) != CUBLAS_STATUS_SUCCESS ||
            cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, k, n, ldb) != CUBLAS_STATUS_SUCCESS ||
            cublasLtMatrixLayoutCreate(&ld, dtype, m, n, ldd) != CUBLAS_STATUS_SUCCESS)
            break;
        if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
        if (cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                                 &ws_bytes, sizeof(ws_bytes)) !=
            CUBLAS_STATUS_SUCCESS)
            break;
        cublasLtMatmulHeuristicResult_t res{};
        int found = 0;
        if (cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, ld, ld, pref, 1, &res, &found) !=
                CUBLAS_STATUS_SUCCESS ||
            found < 1)
            break;
        const float alpha = 1.f;
        ok = cublasLtMatmul(h, op, &alpha, A, la, B, lb, &beta, Dm, ld, Dm, ld, &res.algo, ws,
                            ws_bytes, st) == CUBLAS_STATUS_SUCCESS;
    } while (false);
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (ld) cublasLtMatrixLayoutDestroy(ld);
    if (lb) cublasLtMatrixLayoutDestroy(lb);
    if (la) cublasLtMatrixLayoutDestroy(la);
    if (op) cublasLtMatmulDescDestroy(op);
    return ok;
}

// cat [N][D + Dc] = [x0 | c], rows of bf16 moved as 16-byte chunks (D, Dc multiples of 8)
__global__ void concat_rows_kernel(const uint4* __restrict__ x0, const uint4* __restrict__ c,
                                   uint4* __restrict__ cat, long N, int dq, int cq) {
    const long total = N * (dq + cq);
    for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long)gridDim.x * blockDim.x) {
        const long n = e / (dq + cq);
        const int j = (int)(e - n * (dq + cq));
        cat[e] = j < dq ? x0[n * dq + j] : c[n * cq + (j - dq)];
    }
}

constexpr int kRmsThreads = 256;

__device__ __forceinline__ float rms_block_sum(float x, float* red) {
    x = warp_sum(x);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kRmsThreads / 32; ++w) t += red[w];
    return t;
}

// One CTA per row of D = 8 n fp32 values, n <= kMax * kRmsThreads: each thread keeps up to
// kMax chunks of 8 values in registers (16-byte loads, 16-byte bf16 stores), so the row is
// read once; sum of squares, then the scale and gamma.
template <int kMax>
__global__ void __launch_bounds__(kRmsThreads)
rmsnorm_rows_kernel(const float* __restrict__ z, const float* __restrict__ gamma, float eps,
                    __nv_bfloat16* __restrict__ out, int D) {
    __shared__ float red[kRmsThreads / 32];
    const float* row = z + (size_t)blockIdx.x * D;
    __nv_bfloat16* orow = out + (size_t)blockIdx.x * D;
    const int nch = D / 8;
    float v[kMax][8];
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
        const int ch = threadIdx.x + m * kRmsThreads;
        if (ch < nch) {
            const float4 a = reinterpret_cast<const float4*>(row)[2 * ch];
            const float4 b = reinterpret_cast<const float4*>(row)[2 * ch + 1];
            v[m][0] = a.x; v[m][1] = a.y; v[m][2] = a.z; v[m][3] = a.w;
            v[m][4] = b.x; v[m][5] = b.y; v[m][6] = b.z; v[m][7] = b.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(v[m][e], v[m][e], ss);
        }
    }
    const float inv = rsqrtf(rms_block_sum(ss, red) / (float)D + eps);
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
        const int ch = threadIdx.x + m * kRmsThreads;
        if (ch < nch) {
            float g[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
            if (gamma) {
                const float4 a = reinterpret_cast<const float4*>(gamma)[2 * ch];
                const float4 b = reinterpret_cast<const float4*>(gamma)[2 * ch + 1];
                g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
                g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
            }
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 t = __floats2bfloat162_rn(v[m][2 * e] * inv * g[2 * e],
                                                          v[m][2 * e + 1] * inv * g[2 * e + 1]);
                w[e] = *reinterpret_cast<uint32_t*>(&t);
            }
            reinterpret_cast<uint4*>(orow)[ch] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace

bool gold_gemm_compress(const void* x, const void* w_kd, void* c, long N, int D, int Dc,
                        void* lt_workspace, size_t lt_bytes, cudaStream_t st) {
    // c^T (Dc x N) = w_kd (D x Dc col-major, transposed) . x^T (D x N)
    return gemm_tn(Dc, (int)N, D, w_kd, D, x, D, 0.f, c, CUDA_R_16BF, Dc, lt_workspace,
                   lt_bytes, st);
}

bool gold_gemm_decompress(const void* x0, const void* c, const void* w_ku, void* cat, float* z,
                          long N, int D, int Dc, void* lt_workspace, size_t lt_bytes,
                          cudaStream_t st) {
    const int K = D + Dc, dq = D / 8, cq = Dc / 8;
    const long chunks = N * (dq + cq);
    const unsigned grid = (unsigned)((chunks + 255) / 256 < 148L * 16 ? (chunks + 255) / 256
                                                                       : 148L * 16);
    concat_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(x0),
                                             static_cast<const uint4*>(c),
                                             static_cast<uint4*>(cat), N, dq, cq);
    if (cudaGetLastError() != cudaSuccess) return false;
    // z^T (D x N) = w_ku (K x D col-major, transposed) . cat^T (K x N)
    return gemm_tn(D, (int)N, K, w_ku, K, cat, K, 0.f, z, CUDA_R_32F, D, lt_workspace, lt_bytes,
                   st);
}

cudaError_t launch_rmsnorm_rows(const float* z, const float* gamma, float eps, void* out, long N,
                                int D, cudaStream_t st) {
    if (N <= 0) return cudaSuccess;
    const int per = (D / 8 + kRmsThreads - 1) / kRmsThreads;   // D a multiple of 8
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (per <= 1)
        rmsnorm_rows_kernel<1><<<(unsigned)N, kRmsThreads, 0, st>>>(z, gamma, eps, o, D);
    else if (per <= 2)
        rmsnorm_rows_kernel<2><<<(unsigned)N, kRmsThreads, 0, st>>>(z, gamma, eps, o, D);
    else if (per <= 4)
        rmsnorm_rows_kernel<4><<<(unsigned)N, kRmsThreads, 0, st>>>(z, gamma, eps, o, D);
    else if (per <= 8)
        rmsnorm_rows_kernel<8><<<(unsigned)N, kRmsThreads, 0, st>>>(z, gamma, eps, o, D);
    else
        return cudaErrorInvalidValue;   // D > 16384: not served
    return cudaGetLastError();
}

}  // namespace goldwkv
