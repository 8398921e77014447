// LayerNorm over the concatenated head outputs of each token (Finch-C2 replaces the
// per-head GroupNorm of Finch with one LayerNorm across the full concatenated width;
// GoldFinch review page, section 3.4 "Finch-C2 Time Mixing", output equation):
//     out = (x - mean) / sqrt(var + eps) * gamma + beta,   var = biased variance.
// Used as the second pass after a recurrence kernel has written fp32 rows; one CTA per
// row, exact two-pass mean / variance from the fp32 values.
#include "common.cuh"
#include "internal.h"

namespace goldwkv {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_sum(float x, float* red) {
    x = warp_sum(x);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    return t;
}

template <typename IO>
__global__ void __launch_bounds__(kThreads)
layernorm_rows_kernel(const float* x, const float* __restrict__ gamma,
                      const float* __restrict__ beta, float eps, IO* out, int C) {
    __shared__ float red[kThreads / 32];
    const float* row = x + (size_t)blockIdx.x * C;
    IO* orow = out + (size_t)blockIdx.x * C;
    float s = 0.f;
    for (int c = threadIdx.x; c < C; c += kThreads) s += row[c];
    const float mean = block_sum(s, red) / (float)C;
    float q = 0.f;
    for (int c = threadIdx.x; c < C; c += kThreads) {
        const float d = row[c] - mean;
        q = fmaf(d, d, q);
    }
    const float var = block_sum(q, red) / (float)C;
    const float inv = rsqrtf(var + eps);
    // x and out may alias (fp32 in place): every read of this row happened before the
    // second block_sum's barriers, so overwriting it now is safe.
    for (int c = threadIdx.x; c < C; c += kThreads)
        orow[c] = from_f32<IO>(fmaf((row[c] - mean) * inv, gamma[c], beta[c]));
}

// Base Finch's output normalisation per head, then the output gate (GoldFinch review page,
// section 3.4: Finch-C2 replaces this per-head GroupNorm -- and drops the gate):
//     out = ((x - mean_h) / sqrt(var_h + eps) * gamma + beta) * gate,
// statistics over the D = 64 channels of one head of one token.  One warp per (token, head)
// row, two channels per lane; x may equal out (fp32): a warp reads its row before writing.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
groupnorm_gate_kernel(const float* x, const float* __restrict__ gamma,
                      const float* __restrict__ beta, float eps, const IO* __restrict__ gate,
                      IO* out, long rows, int H) {
    const long row = (long)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, c = 2 * lane;
    const size_t base = (size_t)row * 64;
    const float2 v = *reinterpret_cast<const float2*>(x + base + c);
    const float mean = warp_sum(v.x + v.y) * (1.f / 64.f);
    const float d0 = v.x - mean, d1 = v.y - mean;
    const float var = warp_sum(fmaf(d0, d0, d1 * d1)) * (1.f / 64.f);
    const float inv = rsqrtf(var + eps);
    const int hc = (int)(row % H) * 64 + c;
    float o0 = fmaf(d0 * inv, gamma[hc], beta[hc]);
    float o1 = fmaf(d1 * inv, gamma[hc + 1], beta[hc + 1]);
    if (gate) {
        o0 *= to_f32(gate[base + c]);
        o1 *= to_f32(gate[base + c + 1]);
    }
    out[base + c] = from_f32<IO>(o0);
    out[base + c + 1] = from_f32<IO>(o1);
}

}  // namespace

cudaError_t launch_groupnorm_gate(const float* x, const float* gamma, const float* beta, float eps,
                                  const void* gate, void* out, long rows, int H, bool bf16,
                                  cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kThreads / 32 - 1) / (kThreads / 32));
    if (bf16)
        groupnorm_gate_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
            x, gamma, beta, eps, (const __nv_bfloat16*)gate, (__nv_bfloat16*)out, rows, H);
    else
        groupnorm_gate_kernel<float><<<grid, kThreads, 0, st>>>(
            x, gamma, beta, eps, (const float*)gate, (float*)out, rows, H);
    return cudaGetLastError();
}

cudaError_t launch_layernorm_rows(const float* x, const float* gamma, const float* beta,
                                  float eps, void* out, long rows, int C, bool bf16,
                                  cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    if (bf16)
        layernorm_rows_kernel<__nv_bfloat16><<<(unsigned)rows, kThreads, 0, st>>>(
            x, gamma, beta, eps, (__nv_bfloat16*)out, C);
    else
        layernorm_rows_kernel<float><<<(unsigned)rows, kThreads, 0, st>>>(
            x, gamma, beta, eps, (float*)out, C);
    return cudaGetLastError();
}

}  // namespace goldwkv
