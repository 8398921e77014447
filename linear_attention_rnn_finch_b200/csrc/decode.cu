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
//
// The output stage runs in the same kernel:
//   - base Finch's per-head GroupNorm (+ gate): a head's 64 outputs are in one CTA, which
//     normalises them itself;
//   - Finch-C2's LayerNorm over a token's H*64 outputs (one batch row b): every CTA of the
//     row writes its head's fp32 outputs (to y itself for fp32 I/O, else to the workspace)
//     and counts itself in the row's counter; the CTA that completes the count (the last
//     of the row to finish) reads the row back from L2 and normalises it, then resets the
//     counter to zero.  Nothing waits on another CTA.
#include "common.cuh"
#include "internal.h"

namespace goldwkv {

namespace {

constexpr int kThreads = 256;

enum NormKind { kNoNorm = 0, kLayerNorm = 1, kGroupNorm = 2 };

// Output stage parameters (gamma / beta [H*D] fp32; gate [B][H][D] io or null, GroupNorm
// only; row_count [B] ints, zero between calls, and y_raw [B][H][D] fp32, LayerNorm only)
template <typename IO>
struct OutStage {
    const float* gamma;
    const float* beta;
    float eps;
    const IO* gate;
    int* row_count;
    float* y_raw;
};

__device__ __forceinline__ float block2_sum(float x, float* sbuf, int warp) {
    // sum over the 64 threads of warps 0 and 1 (x from each thread), via one float per warp
    x = warp_sum(x);
    if ((threadIdx.x & 31) == 0) sbuf[warp] = x;
    asm volatile("bar.sync 1, 64;" ::: "memory");
    const float t = sbuf[0] + sbuf[1];
    asm volatile("bar.sync 1, 64;" ::: "memory");
    return t;
}

// uprime != nullptr: Finch-C2 exact form -- key k (1 - w), no static bonus, second value
// u' ([B][H][D], dtype IO) added to y.
template <typename IO, int kNorm>
__global__ void __launch_bounds__(kThreads)
wkv6_decode_kernel(const IO* __restrict__ r, const IO* __restrict__ k,
                   const IO* __restrict__ v, const IO* __restrict__ omega,
                   const float* __restrict__ u, const IO* __restrict__ uprime,
                   float* __restrict__ state, IO* __restrict__ y, OutStage<IO> os, int H) {
    constexpr int D = kHeadSize;
    __shared__ float sr[D], sk[D], sv[D], sw[D];
    __shared__ float4 red[kThreads / 32][D / 4];
    __shared__ float sbonus[2];
    __shared__ float snorm[kThreads / 32 + 2];
    __shared__ int s_last;

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
        if (kNorm == kNoNorm) {
            y[g] = from_f32<IO>(yv);
        } else if (kNorm == kGroupNorm) {
            // this head's 64 outputs: biased variance about the mean, eps inside the root
            const int warp = tid >> 5;
            const float mean = block2_sum(yv, snorm, warp) * (1.f / D);
            const float d = yv - mean;
            const float var = block2_sum(d * d, snorm, warp) * (1.f / D);
            float o = d * rsqrtf(var + os.eps) * os.gamma[h * D + tid] + os.beta[h * D + tid];
            if (os.gate) o *= to_f32(os.gate[g]);
            y[g] = from_f32<IO>(o);
        } else {
            os.y_raw[g] = yv;   // fp32 I/O: y itself
            __threadfence();    // visible device-wide before this CTA is counted
        }
    }
    if (kNorm == kLayerNorm) {
        // count this head in its row; the CTA that completes the count normalises the row
        const int b = bh / H;
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(&os.row_count[b], 1) == H - 1;
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        const int n = H * D;
        const float* row = os.y_raw + (size_t)b * n;
        const int warp = tid >> 5, lane = tid & 31;
        float sum = 0.f;
        for (int i = tid; i < n; i += kThreads) sum += __ldcg(row + i);   // L2: other SMs wrote it
        sum = warp_sum(sum);
        if (lane == 0) snorm[warp] = sum;
        __syncthreads();
        float mean = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) mean += snorm[w];
        mean /= (float)n;
        __syncthreads();
        float sq = 0.f;
        for (int i = tid; i < n; i += kThreads) {
            const float d = __ldcg(row + i) - mean;
            sq = fmaf(d, d, sq);
        }
        sq = warp_sum(sq);
        if (lane == 0) snorm[warp] = sq;
        __syncthreads();
        float var = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) var += snorm[w];
        const float rstd = rsqrtf(var / (float)n + os.eps);
        IO* yrow = y + (size_t)b * n;
        for (int i = tid; i < n; i += kThreads)
            yrow[i] = from_f32<IO>((__ldcg(row + i) - mean) * rstd * os.gamma[i] + os.beta[i]);
        if (tid == 0) os.row_count[b] = 0;   // ready for the next call
    }
}

template <typename IO>
cudaError_t launch_decode_io(const void* r, const void* k, const void* v, const void* omega,
                             const float* u, float* state, void* y, const DecodeOut& out,
                             int B, int H, Variant var, cudaStream_t st) {
    const unsigned grid = (unsigned)(B * H);
    const OutStage<IO> os{out.gamma, out.beta, out.eps, static_cast<const IO*>(out.gate),
                          out.row_count,
                          out.y_raw ? out.y_raw : reinterpret_cast<float*>(y)};
    const IO* args[5] = {(const IO*)r, (const IO*)k, (const IO*)v, (const IO*)omega,
                         (const IO*)var.uprime};
    if (out.kind == 1)
        wkv6_decode_kernel<IO, kLayerNorm><<<grid, kThreads, 0, st>>>(
            args[0], args[1], args[2], args[3], u, args[4], state, (IO*)y, os, H);
    else if (out.kind == 2)
        wkv6_decode_kernel<IO, kGroupNorm><<<grid, kThreads, 0, st>>>(
            args[0], args[1], args[2], args[3], u, args[4], state, (IO*)y, os, H);
    else
        wkv6_decode_kernel<IO, kNoNorm><<<grid, kThreads, 0, st>>>(
            args[0], args[1], args[2], args[3], u, args[4], state, (IO*)y, os, H);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, float* state, void* y, const DecodeOut& out, int B,
                          int H, bool bf16, Variant var, cudaStream_t st) {
    return bf16 ? launch_decode_io<__nv_bfloat16>(r, k, v, omega, u, state, y, out, B, H, var, st)
                : launch_decode_io<float>(r, k, v, omega, u, state, y, out, B, H, var, st);
}

}  // namespace goldwkv
