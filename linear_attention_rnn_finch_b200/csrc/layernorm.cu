// LayerNorm over the concatenated head outputs of each token (Finch-C2 replaces the
// per-head GroupNorm of Finch with one LayerNorm across the full concatenated width;
// GoldFinch review page, section 3.4 "Finch-C2 Time Mixing", output equation):
//     out = (x - mean) / sqrt(var + eps) * gamma + beta,   var = biased variance.
// Used as the second pass after a recurrence kernel has written fp32 rows: a warp per row
// for rows of 512-2048 channels, else one CTA per row; exact two-pass mean / variance from
// the fp32 values (held in registers when the row has at most 8192 channels).  Base Finch's per-head GroupNorm + gate lives here too.
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

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w[e] << 16);
        v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Rows of C = 8 * n channels, n <= kMax * kThreads: each thread holds up to kMax chunks of
// 8 values in registers (16-byte loads and stores), so the row is read from memory once.
template <typename IO, int kMax>
__global__ void __launch_bounds__(kThreads)
layernorm_rows_vec_kernel(const float* x, const float* __restrict__ gamma,
                          const float* __restrict__ beta, float eps, IO* out, int C) {
    __shared__ float red[kThreads / 32];
    const float* row = x + (size_t)blockIdx.x * C;
    IO* orow = out + (size_t)blockIdx.x * C;
    const int nch = C / 8;
    float v[kMax][8];
    float s = 0.f;
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
        const int ch = threadIdx.x + m * kThreads;
        if (ch < nch) {
            load8(row + 8 * ch, v[m]);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += v[m][e];
        }
    }
    const float mean = block_sum(s, red) / (float)C;
    float q = 0.f;
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
        if (threadIdx.x + m * kThreads < nch) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[m][e] -= mean;
                q = fmaf(v[m][e], v[m][e], q);
            }
        }
    }
    const float inv = rsqrtf(block_sum(q, red) / (float)C + eps);
    // x and out may alias (fp32 in place): the row was read before the barriers above
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
        const int ch = threadIdx.x + m * kThreads;
        if (ch < nch) {
            float g[8], b[8];
            load8(gamma + 8 * ch, g);
            load8(beta + 8 * ch, b);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[m][e] = fmaf(v[m][e] * inv, g[e], b[e]);
            store8(orow + 8 * ch, v[m]);
        }
    }
}

// Rows of C = 128 * kV4 channels (at most 2048), one warp per row: lane l holds the row's
// 16-byte pieces l, l + 32, ... in registers, so the row is read from memory once and both
// moments are warp reductions (no block barrier between the steps of a row).  The CTAs are
// persistent, 8 rows at a time, and stage gamma and beta in shared memory once.
__device__ __forceinline__ void store4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
}

constexpr int kRowsPerCta = kThreads / 32;

template <typename IO, int kV4>
__global__ void __launch_bounds__(kThreads)
layernorm_rows_warp_kernel(const float* x, const float* __restrict__ gamma,
                           const float* __restrict__ beta, float eps, IO* out, long rows) {
    constexpr int C = 128 * kV4;
    __shared__ float4 g4[C / 4], b4[C / 4];
    for (int i = threadIdx.x; i < C / 4; i += kThreads) {
        g4[i] = reinterpret_cast<const float4*>(gamma)[i];
        b4[i] = reinterpret_cast<const float4*>(beta)[i];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (long r = (long)blockIdx.x * kRowsPerCta + warp; r < rows;
         r += (long)gridDim.x * kRowsPerCta) {
        const float4* row = reinterpret_cast<const float4*>(x + r * C);
        float4 v[kV4];
#pragma unroll
        for (int m = 0; m < kV4; ++m) v[m] = row[lane + 32 * m];
        float sm = 0.f;
#pragma unroll
        for (int m = 0; m < kV4; ++m) sm += (v[m].x + v[m].y) + (v[m].z + v[m].w);
        const float mean = warp_sum(sm) * (1.f / (float)C);
        float q = 0.f;
#pragma unroll
        for (int m = 0; m < kV4; ++m) {
            v[m].x -= mean; v[m].y -= mean; v[m].z -= mean; v[m].w -= mean;
            q = fmaf(v[m].x, v[m].x, fmaf(v[m].y, v[m].y, fmaf(v[m].z, v[m].z, fmaf(v[m].w, v[m].w, q))));
        }
        const float inv = rsqrtf(warp_sum(q) * (1.f / (float)C) + eps);
        // x and out may alias (fp32 in place): this warp read the whole row above
        IO* orow = out + r * C;
#pragma unroll
        for (int m = 0; m < kV4; ++m) {
            const int i = lane + 32 * m;
            const float4 g = g4[i], b = b4[i];
            store4(orow + 4 * i, fmaf(v[m].x * inv, g.x, b.x), fmaf(v[m].y * inv, g.y, b.y),
                   fmaf(v[m].z * inv, g.z, b.z), fmaf(v[m].w * inv, g.w, b.w));
        }
    }
}

template <typename IO, int kV4>
cudaError_t launch_ln_warp(const float* x, const float* gamma, const float* beta, float eps,
                           IO* out, long rows, cudaStream_t st) {
    const long need = (rows + kRowsPerCta - 1) / kRowsPerCta;
    const unsigned grid = (unsigned)(need < 148L * 8 ? need : 148L * 8);
    layernorm_rows_warp_kernel<IO, kV4><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, out, rows);
    return cudaGetLastError();
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
// statistics over the D = 64 channels of one head of one token.  Eight lanes per (token,
// head) row, eight channels per lane in 16-byte accesses, four rows per warp: short
// per-row dependency chains, so many rows are in flight per SM.  x may equal out (fp32):
// each lane reads its eight values before writing them.
constexpr int kGnLanes = 8;                      // lanes per row
constexpr int kGnRowsPerCta = kThreads / kGnLanes;

__device__ __forceinline__ float gn_sum(float v) {   // over the 8 lanes of a row
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

template <typename IO>
__global__ void __launch_bounds__(kThreads)
groupnorm_gate_kernel(const float* x, const float* __restrict__ gamma,
                      const float* __restrict__ beta, float eps, const IO* __restrict__ gate,
                      IO* out, long rows, int H) {
    // every lane of the warp stays for the shuffles; a group past the last row works on the
    // last row again and does not store
    const long row_id = (long)blockIdx.x * kGnRowsPerCta + (threadIdx.x / kGnLanes);
    const bool valid = row_id < rows;
    const long row = valid ? row_id : rows - 1;
    const int c = 8 * (threadIdx.x % kGnLanes);
    const size_t base = (size_t)row * 64 + c;
    float v[8], g[8], bt[8], gt[8];
    load8(x + base, v);
    const int hc = (int)(row % H) * 64 + c;
    load8(gamma + hc, g);
    load8(beta + hc, bt);
    if (gate) load8(gate + base, gt);
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) sum += v[e];
    const float mean = gn_sum(sum) * (1.f / 64.f);
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        v[e] -= mean;
        sq = fmaf(v[e], v[e], sq);
    }
    const float inv = rsqrtf(gn_sum(sq) * (1.f / 64.f) + eps);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        v[e] = fmaf(v[e] * inv, g[e], bt[e]);
        if (gate) v[e] *= gt[e];
    }
    if (valid) store8(out + base, v);
}

}  // namespace

cudaError_t launch_groupnorm_gate(const float* x, const float* gamma, const float* beta, float eps,
                                  const void* gate, void* out, long rows, int H, bool bf16,
                                  cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kGnRowsPerCta - 1) / kGnRowsPerCta);
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
    // rows of 512, 1024 or 2048 channels (H = 8, 16, 32): a warp per row
    if (C == 512 || C == 1024 || C == 2048) {
        if (bf16) {
            auto* o = (__nv_bfloat16*)out;
            if (C == 512) return launch_ln_warp<__nv_bfloat16, 4>(x, gamma, beta, eps, o, rows, st);
            if (C == 1024) return launch_ln_warp<__nv_bfloat16, 8>(x, gamma, beta, eps, o, rows, st);
            return launch_ln_warp<__nv_bfloat16, 16>(x, gamma, beta, eps, o, rows, st);
        }
        auto* o = (float*)out;
        if (C == 512) return launch_ln_warp<float, 4>(x, gamma, beta, eps, o, rows, st);
        if (C == 1024) return launch_ln_warp<float, 8>(x, gamma, beta, eps, o, rows, st);
        return launch_ln_warp<float, 16>(x, gamma, beta, eps, o, rows, st);
    }
    // C = H * 64: whole 8-value chunks; rows of up to 8192 channels stay in registers
    const int per = (C / 8 + kThreads - 1) / kThreads;
    const unsigned grid = (unsigned)rows;
    if (C % 8 == 0 && per <= 4) {
        if (bf16) {
            auto* o = (__nv_bfloat16*)out;
            if (per == 1) layernorm_rows_vec_kernel<__nv_bfloat16, 1><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
            else if (per == 2) layernorm_rows_vec_kernel<__nv_bfloat16, 2><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
            else layernorm_rows_vec_kernel<__nv_bfloat16, 4><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
        } else {
            auto* o = (float*)out;
            if (per == 1) layernorm_rows_vec_kernel<float, 1><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
            else if (per == 2) layernorm_rows_vec_kernel<float, 2><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
            else layernorm_rows_vec_kernel<float, 4><<<grid, kThreads, 0, st>>>(x, gamma, beta, eps, o, C);
        }
        return cudaGetLastError();
    }
    if (bf16)
        layernorm_rows_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
            x, gamma, beta, eps, (__nv_bfloat16*)out, C);
    else
        layernorm_rows_kernel<float><<<grid, kThreads, 0, st>>>(
            x, gamma, beta, eps, (float*)out, C);
    return cudaGetLastError();
}

}  // namespace goldwkv
