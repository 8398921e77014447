// Token-by-token WKV6 recurrence on CUDA cores, fp32 state and arithmetic.
//
// This is the recursive form of the GoldFinch review page's state sum (section 3.4,
// "Recurrent state update and output"): per (b,h),
//     y_t[j]  = sum_i r_t[i] S[i][j] + (sum_i r_t[i] u[i] k_t[i]) v_t[j]
//     S[i][j] = w_t[i] S[i][j] + k_t[i] v_t[j],   w_t = exp(-exp(omega_t)).
// It serves the fp32-I/O path (tolerance 1e-4) and any shape the chunked tensor-core
// kernel does not take.
//
// Work split: value columns j are independent, so a CTA owns one head and 32 of its 64
// columns (grid = B*H x 2).  Thread (j, q) keeps S[16q..16q+15][j] in registers; the
// readout's sum over i is finished with two xor-shuffles across the four q-threads of a
// column, which sit in adjacent lanes.  Tokens are staged through shared memory in tiles
// of kTile, with w and the per-token bonus coefficient computed once per tile.
#include "common.cuh"
#include "internal.h"

namespace goldwkv {

namespace {

constexpr int kTile = 32;          // tokens staged per shared-memory tile
constexpr int kCols = 32;          // value columns per CTA
constexpr int kThreads = 128;      // 32 columns x 4 row quarters

// uprime != nullptr: Finch-C2 exact form -- key k (1 - w), no static bonus, and the second
// value u'_t (same layout as y) added to the readout.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
wkv6_recurrent_kernel(const IO* __restrict__ r, const IO* __restrict__ k,
                      const IO* __restrict__ v, const IO* __restrict__ omega,
                      const float* __restrict__ u, const IO* __restrict__ uprime,
                      const float* s_in, float* s_out, IO* __restrict__ y,
                      float* __restrict__ y_raw, int T, int H) {
    constexpr int D = kHeadSize;
    __shared__ __align__(16) float sr[kTile][D];
    __shared__ __align__(16) float sk[kTile][D];
    __shared__ __align__(16) float sw[kTile][D];
    __shared__ float sv[kTile][kCols];
    __shared__ float sbonus[kTile];
    __shared__ float su[D];

    const int bh = blockIdx.x;                 // b*H + h
    const int b = bh / H, h = bh - (bh / H) * H;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int q = lane & 3;                    // row quarter: rows 16q .. 16q+15
    const int jl = warp * 8 + (lane >> 2);     // local column 0..31
    const int j = blockIdx.y * kCols + jl;     // global value column

    if (tid < D) su[tid] = uprime ? 0.f : u[h * D + tid];

    // state rows 16q..16q+15 of column j
    float S[16];
    const size_t sbase = (size_t)bh * D * D;
#pragma unroll
    for (int m = 0; m < 16; ++m) S[m] = s_in ? s_in[sbase + (size_t)(16 * q + m) * D + j] : 0.f;

    const size_t tstride = (size_t)H * D;                     // elements between tokens
    const size_t xbase = ((size_t)b * T * H + h) * D;         // (b, t=0, h, 0)

    for (int t0 = 0; t0 < T; t0 += kTile) {
        const int nt = min(kTile, T - t0);
        __syncthreads();  // previous tile fully consumed
        for (int idx = tid; idx < kTile * D; idx += kThreads) {
            const int tt = idx / D, c = idx - (idx / D) * D;
            float rv = 0.f, kv = 0.f, wv = 1.f;
            if (tt < nt) {
                const size_t g = xbase + (size_t)(t0 + tt) * tstride + c;
                rv = to_f32(r[g]);
                kv = to_f32(k[g]);
                wv = decay_from_logit(to_f32(omega[g]));
                if (uprime) kv *= -expm1f(-expf(to_f32(omega[g])));   // k (1 - w)
            }
            sr[tt][c] = rv;
            sk[tt][c] = kv;
            sw[tt][c] = wv;
        }
        for (int idx = tid; idx < kTile * kCols; idx += kThreads) {
            const int tt = idx / kCols, c = idx - (idx / kCols) * kCols;
            sv[tt][c] = tt < nt ? to_f32(v[xbase + (size_t)(t0 + tt) * tstride +
                                          blockIdx.y * kCols + c]) : 0.f;
        }
        __syncthreads();
        // bonus coefficient of each token: sum_i r[i] u[i] k[i]; warp w takes 8 tokens
        for (int tt = warp * (kTile / 4); tt < (warp + 1) * (kTile / 4); ++tt) {
            float p = sr[tt][lane] * su[lane] * sk[tt][lane] +
                      sr[tt][lane + 32] * su[lane + 32] * sk[tt][lane + 32];
            p = warp_sum(p);
            if (lane == 0) sbonus[tt] = p;
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            const float4* r4 = reinterpret_cast<const float4*>(&sr[tt][16 * q]);
            const float4* k4 = reinterpret_cast<const float4*>(&sk[tt][16 * q]);
            const float4* w4 = reinterpret_cast<const float4*>(&sw[tt][16 * q]);
            float acc0 = 0.f, acc1 = 0.f;
            const float vj = sv[tt][jl];
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 rr = r4[m4], kk = k4[m4], ww = w4[m4];
                float* s = &S[4 * m4];
                acc0 = fmaf(rr.x, s[0], acc0);
                acc1 = fmaf(rr.y, s[1], acc1);
                acc0 = fmaf(rr.z, s[2], acc0);
                acc1 = fmaf(rr.w, s[3], acc1);
                s[0] = fmaf(ww.x, s[0], kk.x * vj);
                s[1] = fmaf(ww.y, s[1], kk.y * vj);
                s[2] = fmaf(ww.z, s[2], kk.z * vj);
                s[3] = fmaf(ww.w, s[3], kk.w * vj);
            }
            float acc = acc0 + acc1;
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (q == 0) {
                const size_t g = xbase + (size_t)(t0 + tt) * tstride + j;
                const float yv = fmaf(sbonus[tt], vj, acc) + (uprime ? to_f32(uprime[g]) : 0.f);
                if (y_raw) y_raw[g] = yv;
                else y[g] = from_f32<IO>(yv);
            }
        }
    }

    if (s_out) {
#pragma unroll
        for (int m = 0; m < 16; ++m) s_out[sbase + (size_t)(16 * q + m) * D + j] = S[m];
    }
}

}  // namespace

cudaError_t launch_recurrent(const void* r, const void* k, const void* v, const void* omega,
                             const float* u, const float* s_in, float* s_out, void* y,
                             float* y_raw, int B, int T, int H, bool bf16, Variant var,
                             cudaStream_t st) {
    dim3 grid((unsigned)(B * H), kHeadSize / kCols);
    if (bf16) {
        using T16 = __nv_bfloat16;
        wkv6_recurrent_kernel<T16><<<grid, kThreads, 0, st>>>(
            (const T16*)r, (const T16*)k, (const T16*)v, (const T16*)omega, u,
            (const T16*)var.uprime, s_in, s_out, (T16*)y, y_raw, T, H);
    } else {
        wkv6_recurrent_kernel<float><<<grid, kThreads, 0, st>>>(
            (const float*)r, (const float*)k, (const float*)v, (const float*)omega, u,
            (const float*)var.uprime, s_in, s_out, (float*)y, y_raw, T, H);
    }
    return cudaGetLastError();
}

}  // namespace goldwkv
