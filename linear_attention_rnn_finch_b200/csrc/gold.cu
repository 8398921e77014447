// GOLD key compression and TokenCat decompression (GoldFinch review page, section 3.4 "GOLD
// Key Compression and TokenCat Decompression"):
//     c_t   = x_t W_KD                                   (D -> Dc = D/16)
//     k^D_t = RMSNorm(concat(x0_t, c_t) W_KU)            (D + Dc -> D)
// Both products run in gold_gemm (csrc/gold_gemm_sm100.cu, tcgen05); for D <= 2048 the
// RMSNorm is part of that kernel's epilogue.  This file keeps the row-wise RMSNorm used
// when D is wider than one thread-block cluster of column tiles: the product is then
// written as fp32 and normalised here.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gold.h"

namespace goldwkv {

namespace {

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
