// One autoregressive WKV6 step (T = 1) with the fp32 state updated in place.
//
// Per (b,h) (GoldFinch review page, section 3.4, "Recurrent state update and output",
// one token of the recurrence; "Training and Inference Procedures": the recurrent layers
// take each generated token in O(1)):
//     y[j]    = sum_i r[i] S[i][j] + (sum_i r[i] u[i] k[i]) v[j]
//     S[i][j] = w[i] S[i][j] + k[i] v[j],    w = exp(-exp(omega)).
//
// The step is a pure stream over the 16 KB state of each head, so the kernel is shaped
// for HBM: one 256-thread CTA per head, every thread moves four 16-byte vectors of the
// state (rows r0, r0+16, r0+32, r0+48; columns 4c..4c+3) with streaming cache hints, a
// warp's load instruction covers two full 256-byte rows, and the loads are issued before
// the small r/k/v/omega staging so their latency overlaps it.
#include "common.cuh"
#include "internal.h"

namespace goldwkv {

namespace {

constexpr int kThreads = 256;

// uprime != nullptr: Finch-C2 exact form -- key k (1 - w), no static bonus, second value
// u' ([B][H][D], dtype IO) added to y.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
wkv6_decode_kernel(const IO* __restrict__ r, const IO* __restrict__ k,
                   const IO* __restrict__ v, const IO* __restrict__ omega,
                   const float* __restrict__ u, const IO* __restrict__ uprime,
                   float* __restrict__ state, IO* __restrict__ y, float* __restrict__ y_raw,
                   int H) {
    constexpr int D = kHeadSize;
    __shared__ float sr[D], sk[D], sv[D], sw[D];
    __shared__ float4 red[kThreads / 32][D / 4];
    __shared__ float sbonus[2];

    const int bh = blockIdx.x;
    const int h = bh % H;
    const int tid = threadIdx.x;
    const int c = tid & 15;            // column group: j = 4c .. 4c+3
    const int r0 = tid >> 4;           // row block: rows r0 + 16m
    float4* S = reinterpret_cast<float4*>(state + (size_t)bh * D * D);

    float4 s[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) s[m] = __ldcs(&S[(r0 + 16 * m) * (D / 4) + c]);

    if (tid < D) {
        const size_t g = (size_t)bh * D + tid;
        const float rv = to_f32(r[g]), om = to_f32(omega[g]);
        float kv = to_f32(k[g]);
        if (uprime) kv *= -expm1f(-expf(om));   // k (1 - w)
        sr[tid] = rv;
        sk[tid] = kv;
        sv[tid] = to_f32(v[g]);
        sw[tid] = decay_from_logit(om);
        const float p = uprime ? 0.f : warp_sum(rv * u[h * D + tid] * kv);
        if ((tid & 31) == 0) sbonus[tid >> 5] = p;
    }
    __syncthreads();

    const float4 vj = reinterpret_cast<const float4*>(sv)[c];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = r0 + 16 * m;
        const float ri = sr[i], ki = sk[i], wi = sw[i];
        float4 x = s[m];
        acc.x = fmaf(ri, x.x, acc.x);
        acc.y = fmaf(ri, x.y, acc.y);
        acc.z = fmaf(ri, x.z, acc.z);
        acc.w = fmaf(ri, x.w, acc.w);
        x.x = fmaf(wi, x.x, ki * vj.x);
        x.y = fmaf(wi, x.y, ki * vj.y);
        x.z = fmaf(wi, x.z, ki * vj.z);
        x.w = fmaf(wi, x.w, ki * vj.w);
        __stcs(&S[i * (D / 4) + c], x);
    }
    // rows r0 = 2*warp and 2*warp+1 share a warp: fold them, then across warps via smem
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
    if ((tid & 31) < 16) red[tid >> 5][c] = acc;
    __syncthreads();
    if (tid < D) {
        const float* redf = reinterpret_cast<const float*>(red);
        float yv = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) yv += redf[w * D + tid];
        yv = fmaf(sbonus[0] + sbonus[1], sv[tid], yv);
        const size_t g = (size_t)bh * D + tid;
        if (uprime) yv += to_f32(uprime[g]);
        if (y_raw) y_raw[g] = yv;
        else y[g] = from_f32<IO>(yv);
    }
}

}  // namespace

cudaError_t launch_decode(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, float* state, void* y, float* y_raw, int B, int H,
                          bool bf16, Variant var, cudaStream_t st) {
    const unsigned grid = (unsigned)(B * H);
    if (bf16) {
        using T16 = __nv_bfloat16;
        wkv6_decode_kernel<T16><<<grid, kThreads, 0, st>>>(
            (const T16*)r, (const T16*)k, (const T16*)v, (const T16*)omega, u,
            (const T16*)var.uprime, state, (T16*)y, y_raw, H);
    } else {
        wkv6_decode_kernel<float><<<grid, kThreads, 0, st>>>(
            (const float*)r, (const float*)k, (const float*)v, (const float*)omega, u,
            (const float*)var.uprime, state, (float*)y, y_raw, H);
    }
    return cudaGetLastError();
}

}  // namespace goldwkv
