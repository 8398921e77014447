// dr of the WKV6 backward on the tensor cores (sm_100a): the chunked form of the readout of
// the forward state with dy as the query.
//
// Forward (GoldFinch review page, section 3.4 "Recurrent state update and output"), per (b,h):
//     S_t = diag(w_t) S_{t-1} + k_t^T v_t,   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),
// so dr_t[i] = sum_j S_{t-1}[i][j] dy_t[j] + u[i] k_t[i] (v_t . dy_t), the first term a
// readout of the forward state in which the decay sits on the output index i.  For a chunk of
// C = 64 tokens entering with state S, with L_t = sum_{tau<=t} log2 w_tau inside the chunk:
//     S_{t-1}[i][j] = 2^(L_{t-1}[i]) S[i][j] + sum_{s<t} 2^(L_{t-1}[i] - L_s[i]) k_s[i] v_s[j]
//     dr_t[i] = F[t][i] (Z[t][i] + sum_{s<t} A[t][s] Kh[s][i]) + u[i] k_t[i] A[t][t]
// with  F[t][i] = 2^(L_{t-1}[i]) <= 1,  Kh[s][i] = k_s[i] 2^(-L_s[i]),  A = dy v^T (the scores,
// no decay), Z = dy S^T.  The one-sided factor Kh is bounded by 2^86.56 when every channel's
// log2 decay over the chunk is >= -86.56; a (b,h) with a chunk outside that range is flagged
// and left to the CUDA-core scan (fallback[bh] = 1), which redoes its whole sequence.
// The state itself advances with the suffix factors Kt_s = k_s 2^(L_{C-1} - L_s) <= 1 (any
// decay): S <- diag(2^L_{C-1}) S + Kt^T V.
//
// Steps of a chunk (one CTA per (b,h), 256 threads, all warps in lockstep):
//   prep  : warp = 8 channels, lane = 2 tokens; log2 w, the prefix L by a warp scan, F (fp32),
//           Kh and Kt^T as bf16 hi / lo tiles, gamma;
//   MMA 1 : A = dy x v^T; Z = dy x [S_hi ; S_lo]^T (N = 128); U = Kt_hi^T V + Kt_lo^T V;
//   A     : strictly causal part, hi / lo tiles; the diagonal (v_t . dy_t) kept aside;
//   MMA 2 : Z += A_hi [Kh_hi | Kh_lo] + A_lo [Kh_hi | Kh_lo] (N = 128); the output adds Z's
//           two 64-column halves;
//   state : S <- gamma S + U in registers, S_hi / S_lo tiles for the next chunk;
//   out   : dr = F Z + u k diag (bf16 tile, TMA store); for the decay gradient the pair
//           terms ending at t, P_t = r_t (dr_t - bonus) (fp32), and du's per-(b,h) sums.
// The M = 64 accumulators (A, U, Z) keep their rows in lanes 0-15 of each TMEM
// sub-partition; a two-half TMEM load gives every thread of a warp a row, 16 columns each,
// so the A, state and out steps run on all 32 lanes (the state S too: 16 fp32 a thread).
// Pipelined over chunks: iteration n forms A(n), issues MMA 2(n), advances the state and
// prepares chunk n+1 while MMA 2 runs, issues MMA 1(n+1), and forms the output of n while
// MMA 1(n+1) runs (prep buffers, F, gamma and Z alternate by chunk parity).
// At the end: E[i] = sum_j S_T[i][j] dS_T[i][j] (with the dk scan's decay gradient) and du.
// P, E and du_part have the layout and meaning of the CUDA-core dr scan's (csrc/backward.cu).
//
// dk is the same computation in reversed time (kDk): with G_{t-1} = diag(w_t) G_t + r_t^T dy_t
// the state gradient, dk_t[i] = sum_j G_t[i][j] v_t[j] + u[i] r_t[i] (v_t . dy_t), i.e. the
// readout above on time-reversed copies with query v, key r, value dy, initial state dS_T;
// its final state is dS_0, and its pair terms Q_t = k_t (dk_t - bonus) feed the decay
// gradient (wkv6_bwd_domega kernels below).
//
// Finch-C2's exact form (kC2): the key enters the state as kn = k (1 - w) and there is no
// bonus.  dr: the key is kn, formed in prep.  dk: the readout is dkn (the key of the reversed
// recurrence is r, unchanged); dk = dkn (1 - w), Q_t = kn_t dkn_t, and kn's own dependence on
// w adds D_t = dkn_t k_t w_t, subtracted from dlog w_t.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "backward.h"
#include "chunk_tiles.cuh"
#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kTile = 64 * 64 * 2;
constexpr uint32_t kTmemCols = 512;
// Z: 2 x 128 (chunk parity; the S_hi / Kh_hi part in the first 64 columns, the lo part next)
constexpr uint32_t COL_A = 0, COL_U = 64, COL_Z = 128;
constexpr uint32_t IDESC_KK = ptx::idesc_bf16(64, 64, 0, 0);
constexpr uint32_t IDESC_KM = ptx::idesc_bf16(64, 64, 0, 1);
constexpr uint32_t IDESC_KK2 = ptx::idesc_bf16(64, 128, 0, 0);   // B = two tiles side by side in N
constexpr uint32_t IDESC_KM2 = ptx::idesc_bf16(64, 128, 0, 1);
constexpr float kMaxLog2Range = 86.5617f;   // ln 60
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kFPitch = 68;                 // floats per row of F (padded against bank conflicts)

struct __align__(1024) Smem {
    uint8_t in[kStages][4][kTile];   // dy, k, v, omega tiles per stage (TMA, 128B swizzle)
    uint8_t kh[2][2][kTile];                // Kh [s][i] per chunk parity: hi tile, then lo tile
    uint8_t kt_hi[2][kTile], kt_lo[2][kTile];   // Kt^T [i][s], per chunk parity
    uint8_t a_hi[kTile], a_lo[kTile];       // causal scores [t][s]
    uint8_t s_hi[kTile], s_lo[kTile];       // S [i][j]
    uint8_t ystage[2][kTile];               // dr tiles for the TMA store
    float F[2][C][kFPitch];                 // per chunk parity
    float u[64];
    float gamma[2][64];
    float diag[64];                         // v_t . dy_t
    float epart[2][64];                     // E halves
    float dupart[4][64];                    // du sums per row quarter
    uint64_t full[kStages];
    uint64_t mma1, mma2;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t sw_chunk(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}
// hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split8(const float (&f)[8], uint4& hi, uint4& lo) {
    float h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = __bfloat162float(__float2bfloat16_rn(f[i]));
        l[i] = f[i] - h[i];
    }
    hi = pack8(h);
    lo = pack8(l);
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// the two bf16 of a transposed tile entry: channel row i, tokens (2 lane, 2 lane + 1)
__device__ __forceinline__ uint32_t tr_off(int i, int lane) {
    return (uint32_t)(i * 128 + ((((lane >> 2)) ^ (i & 7)) << 4) + (lane & 3) * 4);
}

// kDk == false (dr): query dy, key k, value v, aux r, x0 = state_in; writes P, E, du_part.
// kDk == true (dk, time-reversed inputs): query v, key r, value dy, aux k (in token order),
// x0 = dS_T; writes dk to out_direct and Q (into P), both in token order, and the final state
// (dS_0) to x_final.
template <bool kDk, bool kC2>
__global__ void __launch_bounds__(kThreads, 1)
wkv6_bwd_readout_tc_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_dr, const __nv_bfloat16* __restrict__ r,
                      const float* __restrict__ u, const float* state_in, const float* dS_T,
                      float* __restrict__ P, float* __restrict__ E, float* __restrict__ du_part,
                      float* x_final, __nv_bfloat16* __restrict__ out_direct,
                      float* __restrict__ Dw, int* fallback, int T,
                      int H, int* status, long long budget, long long drain_budget) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x, b = bh / H, h = bh - (bh / H) * H;
    const int NC = (T + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) ptx::mbar_init(&s.full[i], 1);
        ptx::mbar_init(&s.mma1, 1);
        ptx::mbar_init(&s.mma2, 1);
        ptx::fence_mbar_init();
        s.abort = 0;
        ptx::prefetch_tensormap(&tm_dy);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_w);
        ptx::prefetch_tensormap(&tm_dr);
    }
    if (tid < 64) s.u[tid] = kC2 ? 0.f : u[h * 64 + tid];
    if (warp == 0) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    auto issue_load = [&](int n) {
        const int st = n % kStages, t0 = n * C;
        if (!gw_check(status, n >= 0 && n < NC && t0 < T && h < H)) return;
        ptx::mbar_arrive_expect_tx(&s.full[st], 4 * kTile);
        ptx::tma_load_4d(s.in[st][0], &tm_dy, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][1], &tm_k, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][2], &tm_v, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][3], &tm_w, &s.full[st], 0, h, t0, b);
    };
    if (tid == 0)
        for (int n = 0; n < kStages && n < NC; ++n) issue_load(n);

    // warp w: TMEM sub-partition q = w % 4 (rows 16q .. 16q+15 in its lanes 0..15), columns
    // 32 hh .. 32 hh + 31.  Lane l takes row 16q + (l & 15) and 16 of those columns, from
    // cb = 32 hh + 16 (l >> 4): the two-half TMEM load gives every lane a row.
    const int q = warp & 3, hh = warp >> 2;
    const int row = 16 * q + (lane & 15);        // state row i / token row t of this lane
    const int cb = 32 * hh + 16 * (lane >> 4);   // its first column
    const int cc0 = cb >> 3;                     // its first 16-byte chunk of a tile row
    const uint32_t tlane = (uint32_t)(32 * q) << 16;
    float S[16];
    {
        const float* src = state_in ? state_in + (size_t)bh * 4096 + row * 64 + cb : nullptr;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (src) x = *reinterpret_cast<const float4*>(src + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = S[8 * cc + e];
            uint4 hi, lo;
            split8(f, hi, lo);
            *reinterpret_cast<uint4*>(s.s_hi + sw_chunk(row, cc0 + cc)) = hi;
            *reinterpret_cast<uint4*>(s.s_lo + sw_chunk(row, cc0 + cc)) = lo;
        }
    }
    float du_acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) du_acc[j] = 0.f;

    bool failed = false, out_of_range = false;
    int issued1 = -1, issued2 = -1;
    int last_load[kStages] = {-1, -1};   // latest chunk whose copy each stage received
    if (tid == 0)
        for (int m = 0; m < kStages && m < NC; ++m) last_load[m] = m;

    // prep of chunk m into the buffers of parity m & 1 (all threads); false if a channel's
    // log2 decay over the chunk is below -86.56
    auto prep_chunk = [&](int m) -> bool {
        const int st = m % kStages, pb = m & 1, valid = min(C, T - m * C);
        const uint8_t* k_tile = s.in[st][1];
        const uint8_t* w_tile = s.in[st][3];
        const int cg = warp;                    // channels 8cg .. 8cg+7
        const int ta = 2 * lane, tb = ta + 1;   // tokens of this lane
        float kv[2][8], lw[2][8];
        {
            float om[2][8];
            unpack8(*reinterpret_cast<const uint4*>(k_tile + sw_chunk(ta, cg)), kv[0]);
            unpack8(*reinterpret_cast<const uint4*>(k_tile + sw_chunk(tb, cg)), kv[1]);
            unpack8(*reinterpret_cast<const uint4*>(w_tile + sw_chunk(ta, cg)), om[0]);
            unpack8(*reinterpret_cast<const uint4*>(w_tile + sw_chunk(tb, cg)), om[1]);
            float ew[2][8];   // exp(omega)
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                for (int c = 0; c < 8; ++c) {   // log2 w = -exp(omega) log2(e); 0 past T
                    ew[q2][c] = ex2(om[q2][c] * kLog2e);
                    lw[q2][c] = (ta + q2 < valid) ? -ew[q2][c] * kLog2e : 0.f;
                }
            if (kC2 && !kDk) {   // the state's key is kn = k (1 - w), 1 - w = 1 - exp(-exp(omega))
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {
                        const float2 f = tiles::one_minus_exp_neg2(make_float2(ew[q2][c], ew[q2][c + 1]));
                        const bool in = ta + q2 < valid;
                        kv[q2][c] *= in ? f.x : 0.f;
                        kv[q2][c + 1] *= in ? f.y : 0.f;
                    }
            }
        }
        // inclusive prefix over the chunk: this lane's pair, then a scan over the lanes
        float inc[8], L63[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) inc[c] = lw[0][c] + lw[1][c];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float o = __shfl_up_sync(0xffffffffu, inc[c], d);
                if (lane >= d) inc[c] += o;
            }
        }
        bool ok = true;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            L63[c] = __shfl_sync(0xffffffffu, inc[c], 31);
            ok = ok && L63[c] >= -kMaxLog2Range;
        }
        if (!ok) return false;
        // L of the two tokens (inclusive) and of the token before each (exclusive)
        float Lt[2][8], Lx[2][8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            Lt[1][c] = inc[c];
            Lt[0][c] = inc[c] - lw[1][c];
            Lx[1][c] = Lt[0][c];
            Lx[0][c] = Lt[0][c] - lw[0][c];
        }
        float khf[2][8];   // Kh in fp32, kept for Kt below
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            float f[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                khf[q2][c] = kv[q2][c] * ex2(-Lt[q2][c]);
                f[c] = ex2(Lx[q2][c]);
            }
            uint4 hi, lo;
            split8(khf[q2], hi, lo);
            *reinterpret_cast<uint4*>(s.kh[pb][0] + sw_chunk(ta + q2, cg)) = hi;
            *reinterpret_cast<uint4*>(s.kh[pb][1] + sw_chunk(ta + q2, cg)) = lo;
            float4* fd = reinterpret_cast<float4*>(&s.F[pb][ta + q2][8 * cg]);
            fd[0] = make_float4(f[0], f[1], f[2], f[3]);
            fd[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
        // Kt = k 2^(L63 - L) = Kh * gamma: both factors are within the range test's bounds
        // (2^(-L) <= 2^86.56, gamma >= 2^-86.56), so the product is a normal fp32 number
        float gam[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) gam[c] = ex2(L63[c]);
#pragma unroll
        for (int c = 0; c < 8; ++c) {   // Kt^T: channel row i, this lane's two tokens
            const int i = 8 * cg + c;
            const float x0 = khf[0][c] * gam[c];
            const float x1 = khf[1][c] * gam[c];
            const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
            const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
            *reinterpret_cast<uint32_t*>(s.kt_hi[pb] + tr_off(i, lane)) = pack2(h0, h1);
            *reinterpret_cast<uint32_t*>(s.kt_lo[pb] + tr_off(i, lane)) = pack2(x0 - h0, x1 - h1);
        }
        if (lane == 0)
#pragma unroll
            for (int c = 0; c < 8; ++c) s.gamma[pb][8 * cg + c] = gam[c];
        return true;
    };
    // MMA 1 of chunk m (one thread): A = dy v^T, Z[m & 1] = dy S^T (S = the state entering m,
    // in s_hi / s_lo), U = Kt^T V
    auto issue_mma1 = [&](int m) {
        const int st = m % kStages, pb = m & 1;
        ptx::tc_fence_after();
        const uint32_t a_dy = ptx::smem_addr(s.in[st][0]), b_v = ptx::smem_addr(s.in[st][2]);
        const uint32_t b_s = ptx::smem_addr(s.s_hi);   // s_lo follows: [S_hi ; S_lo] in N
        const uint32_t a_kh = ptx::smem_addr(s.kt_hi[pb]), a_kl = ptx::smem_addr(s.kt_lo[pb]);
        const uint32_t zc = tmem + COL_Z + 128 * pb;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)   // A = dy v^T
            ptx::mma_bf16(tmem + COL_A, ptx::desc_kmajor(a_dy + 32 * kq),
                          ptx::desc_kmajor(b_v + 32 * kq), IDESC_KK, kq > 0);
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)   // Z = dy [S_hi ; S_lo]^T (the two parts in N)
            ptx::mma_bf16(zc, ptx::desc_kmajor(a_dy + 32 * kq), ptx::desc_kmajor(b_s + 32 * kq),
                          IDESC_KK2, kq > 0);
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)   // U = Kt_hi^T V
            ptx::mma_bf16(tmem + COL_U, ptx::desc_kmajor(a_kh + 32 * kq),
                          ptx::desc_mnmajor(b_v + 2048 * kq), IDESC_KM, kq > 0);
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)   // U += Kt_lo^T V
            ptx::mma_bf16(tmem + COL_U, ptx::desc_kmajor(a_kl + 32 * kq),
                          ptx::desc_mnmajor(b_v + 2048 * kq), IDESC_KM, 1);
        ptx::mma_commit(&s.mma1);
        issued1 = m;
    };

    // Software pipeline over chunks, all threads in lockstep: MMA 2 of chunk n runs while the
    // state advances and chunk n+1 is prepared; MMA 1 of chunk n+1 runs while chunk n's
    // output is formed.
    int n = 0;
    {
        if (!ptx::mbar_wait(&s.full[0], 0, budget)) s.abort = 1;
        const bool ok = NC > 0 && prep_chunk(0);
        ptx::fence_proxy_async_smem();
        if (__syncthreads_or(!ok || s.abort)) {
            if (s.abort) failed = true;
            else out_of_range = true;
        } else if (tid == 0) {
            issue_mma1(0);
        }
    }
    if (!failed && !out_of_range) for (; n < NC; ++n) {
        const int st = n % kStages, pb = n & 1;
        const int t0 = n * C;
        const int valid = min(C, T - t0);
        uint8_t* k_tile = s.in[st][1];
        uint8_t* y_tile = s.ystage[pb];
        // the aux row (r, or k in reversed time) of this lane, read now for the output step
        const int t = row;
        const bool live = t < valid;
        // this row in the caller's token order: dk's inputs are time-reversed, its outputs
        // (dk, Q) and its aux input (k) are not
        const int tok = kDk ? T - 1 - (t0 + t) : t0 + t;
        const size_t gx = (((size_t)b * T + tok) * H + h) * 64 + cb;
        uint4 rw[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
            rw[cc] = live ? __ldg(reinterpret_cast<const uint4*>(r + gx + 8 * cc)) : make_uint4(0, 0, 0, 0);
        // the store that last used y_tile (chunk n-2) has read it before this chunk rewrites it
        if (!kDk && tid == 0) ptx::bulk_wait_read<1>();

        if (!ptx::mbar_wait(&s.mma1, (uint32_t)(n & 1), budget)) s.abort = 1;
        ptx::tc_fence_after();
        // -------------------------------------------------------- causal scores of chunk n
        {
            uint32_t A[16];
            ptx::tmem_ld16x2(tmem + tlane + COL_A + 32 * hh, A);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int sx = cb + 8 * cc + e;
                    const float x = __uint_as_float(A[8 * cc + e]);
                    if (sx == t) s.diag[t] = x;
                    a[e] = sx < t ? x : 0.f;
                }
                uint4 hi, lo;
                split8(a, hi, lo);
                *reinterpret_cast<uint4*>(s.a_hi + sw_chunk(t, cc0 + cc)) = hi;
                *reinterpret_cast<uint4*>(s.a_lo + sw_chunk(t, cc0 + cc)) = lo;
            }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        // (a vote, not a read after the barrier: a thread already past it may set abort)
        if (__syncthreads_or(s.abort)) { failed = true; break; }
        // -------------------------------------------------------- MMA 2: Z[n & 1] += A Kh
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t ah = ptx::smem_addr(s.a_hi), al = ptx::smem_addr(s.a_lo);
            const uint32_t bk = ptx::smem_addr(s.kh[pb][0]);   // [Kh_hi | Kh_lo] in N
            const uint32_t zc = tmem + COL_Z + 128 * pb;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)   // Z += A_hi [Kh_hi | Kh_lo]
                ptx::mma_bf16(zc, ptx::desc_kmajor(ah + 32 * kq), ptx::desc_sw128(bk + 2048 * kq, kTile),
                              IDESC_KM2, 1);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)   // Z += A_lo [Kh_hi | Kh_lo]
                ptx::mma_bf16(zc, ptx::desc_kmajor(al + 32 * kq), ptx::desc_sw128(bk + 2048 * kq, kTile),
                              IDESC_KM2, 1);
            ptx::mma_commit(&s.mma2);
            issued2 = n;
        }
        // -------------------------------------------------------- state chain (MMA 2 running)
        {
            uint32_t U[16];
            ptx::tmem_ld16x2(tmem + tlane + COL_U + 32 * hh, U);
            ptx::tmem_wait_ld();
            const float g = s.gamma[pb][row];
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(g, S[j], __uint_as_float(U[j]));
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = S[8 * cc + e];
                uint4 hi, lo;
                split8(f, hi, lo);
                *reinterpret_cast<uint4*>(s.s_hi + sw_chunk(row, cc0 + cc)) = hi;
                *reinterpret_cast<uint4*>(s.s_lo + sw_chunk(row, cc0 + cc)) = lo;
            }
        }
        // -------------------------------------------------------- prep of chunk n+1
        bool next_ok = true;
        if (n + 1 < NC) {
            if (!ptx::mbar_wait(&s.full[(n + 1) % kStages], (uint32_t)(((n + 1) / kStages) & 1), budget))
                s.abort = 1;
            next_ok = prep_chunk(n + 1);
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        const bool stop = __syncthreads_or(!next_ok || s.abort);
        // MMA 1 of chunk n+1 (its inputs, the S tiles above and its operands, are in place;
        // A and U of chunk n have been read)
        if (!stop && tid == 0 && n + 1 < NC) issue_mma1(n + 1);
        if (!ptx::mbar_wait(&s.mma2, (uint32_t)(n & 1), budget)) s.abort = 1;
        ptx::tc_fence_after();
        // -------------------------------------------------------- output of chunk n
        {
            uint32_t Z[16], Z2[16];
            ptx::tmem_ld16x2(tmem + tlane + COL_Z + 128 * pb + 32 * hh, Z);
            ptx::tmem_ld16x2(tmem + tlane + COL_Z + 128 * pb + 64 + 32 * hh, Z2);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) Z[j] = __float_as_uint(__uint_as_float(Z[j]) + __uint_as_float(Z2[j]));
            {
                const float dg = s.diag[t];
                float* pdst = P + gx;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float kx[8], o[8], pv[8], rv[8], dv8[8];
                    unpack8(*reinterpret_cast<const uint4*>(k_tile + sw_chunk(t, cc0 + cc)), kx);
                    unpack8(rw[cc], rv);
                    float om[8], omw8[8], w8[8];
                    if (kC2 && kDk) {   // this token's omega (reversed-time tile, row t)
                        unpack8(*reinterpret_cast<const uint4*>(s.in[st][3] + sw_chunk(t, cc0 + cc)), om);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {   // w and 1 - w of x = exp(omega)
                            const float2 x = make_float2(ex2(om[e] * kLog2e), ex2(om[e + 1] * kLog2e));
                            const float2 f = tiles::one_minus_exp_neg2(x);
                            omw8[e] = f.x;
                            omw8[e + 1] = f.y;
                            w8[e] = ex2(-x.x * kLog2e);
                            w8[e + 1] = ex2(-x.y * kLog2e);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 8 * cc + e, i = cb + j;
                        const float pair = s.F[pb][t][i] * __uint_as_float(Z[j]);   // minus the bonus
                        if (kC2 && kDk) {
                            // pair = dkn; dk = dkn (1 - w); Q = kn dkn = k (1 - w) dkn; D = dkn k w
                            const float omw = omw8[e], w = w8[e];
                            o[e] = pair * omw;
                            pv[e] = rv[e] * omw * pair;
                            dv8[e] = pair * rv[e] * w;
                        } else {
                            const float kd = kx[e] * dg;
                            o[e] = fmaf(s.u[i], kd, pair);
                            pv[e] = rv[e] * pair;
                            du_acc[j] = fmaf(rv[e], kd, du_acc[j]);
                        }
                    }
                    if (!kDk)
                        *reinterpret_cast<uint4*>(y_tile + sw_chunk(t, cc0 + cc)) = pack8(o);
                    else if (live)   // dk straight to its row in token order
                        *reinterpret_cast<uint4*>(out_direct + gx + 8 * cc) = pack8(o);
                    if (live) {
                        reinterpret_cast<float4*>(pdst + 8 * cc)[0] = make_float4(pv[0], pv[1], pv[2], pv[3]);
                        reinterpret_cast<float4*>(pdst + 8 * cc)[1] = make_float4(pv[4], pv[5], pv[6], pv[7]);
                        if (kC2 && kDk) {
                            reinterpret_cast<float4*>(Dw + gx + 8 * cc)[0] = make_float4(dv8[0], dv8[1], dv8[2], dv8[3]);
                            reinterpret_cast<float4*>(Dw + gx + 8 * cc)[1] = make_float4(dv8[4], dv8[5], dv8[6], dv8[7]);
                        }
                    }
                }
            }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        const bool brk = __syncthreads_or(stop || s.abort);
        if (tid == 0) {
            if (!kDk && gw_check(status, t0 < T && h < H)) {
                ptx::tma_store_4d(&tm_dr, y_tile, 0, h, t0, b);
                ptx::bulk_commit();
            }
            // every thread is past its reads of stage st and the MMAs that read it are done
            if (!brk && n + kStages < NC) {
                ptx::fence_proxy_async_smem();
                issue_load(n + kStages);
                last_load[st] = n + kStages;
            }
        }
        if (brk) {   // every abort write precedes the vote, so all threads read the same
            if (s.abort) failed = true;
            else out_of_range = true;
            ++n;   // chunk n is complete; the drain below starts after it
            break;
        }
    }

    // ------------------------------------------------------------ finish / drain
    if (failed || out_of_range) {
        if (tid == 0) {
            if (failed) atomicExch(status, 1);
            // every issued copy must land (waiting again on a landed one returns at once),
            // and the products of the chunk this CTA stopped at must be complete
            for (int st = 0; st < kStages; ++st)
                if (last_load[st] >= 0)
                    ptx::mbar_wait(&s.full[st], (uint32_t)((last_load[st] / kStages) & 1), drain_budget);
            if (issued1 == n) ptx::mbar_wait(&s.mma1, (uint32_t)(n & 1), drain_budget);
            if (issued2 == n) ptx::mbar_wait(&s.mma2, (uint32_t)(n & 1), drain_budget);
            fallback[bh] = 1;   // the CUDA-core scan redoes this (b,h)
        }
    } else if (kDk) {
        if (x_final != nullptr) {   // dS_0
            float* dst = x_final + (size_t)bh * 4096 + row * 64 + cb;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (tid == 0) fallback[bh] = 0;
    } else {
        // E[i] = sum_j S_T[i][j] dS_T[i][j]; du[i] = sum_t r_t[i] k_t[i] (v_t . dy_t)
        float ev = 0.f;
        if (dS_T) {
            const float* g = dS_T + (size_t)bh * 4096 + row * 64 + cb;
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(g + j);
                ev = fmaf(S[j], x.x, fmaf(S[j + 1], x.y, fmaf(S[j + 2], x.z, fmaf(S[j + 3], x.w, ev))));
            }
        }
        ev += __shfl_xor_sync(0xffffffffu, ev, 16);   // the row's other 16 columns
        if (lane < 16) s.epart[hh][row] = ev;
        // du: sum over the 16 row lanes of each half-warp, then over the 4 row quarters
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float x = du_acc[j];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            du_acc[j] = x;
        }
        if ((lane & 15) == 0)
#pragma unroll
            for (int j = 0; j < 16; ++j) s.dupart[q][cb + j] = du_acc[j];
        __syncthreads();
        if (tid < 64) {
            E[(size_t)bh * 64 + tid] = s.epart[0][tid] + s.epart[1][tid];
            du_part[(size_t)bh * 64 + tid] =
                s.dupart[0][tid] + s.dupart[1][tid] + s.dupart[2][tid] + s.dupart[3][tid];
        }
        if (tid == 0) fallback[bh] = 0;
    }
    if (tid == 0) ptx::bulk_wait<0>();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

size_t bwd_readout_tc_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_bwd_dr_tc(const CUtensorMap* maps, const void* r, const float* u,
                             const float* state_in, const float* dS_T, float* P, float* E,
                             float* du_part, int* fallback, int B, int T, int H, int* status,
                             long long budget, cudaStream_t st, bool c2) {
    const size_t smem = bwd_readout_tc_smem_bytes();
    auto kernel = c2 ? wkv6_bwd_readout_tc_kernel<false, true> : wkv6_bwd_readout_tc_kernel<false, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)(B * H), kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], static_cast<const __nv_bfloat16*>(r), u,
        state_in, dS_T, P, E, du_part, nullptr, nullptr, nullptr, fallback, T, H, status, budget,
        4000000000LL);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dk_tc(const CUtensorMap* maps, const void* k, const float* u,
                             const float* dS_T, void* dk, float* Q, float* D, float* dS_0,
                             int* fallback, int B, int T, int H, int* status, long long budget,
                             cudaStream_t st, bool c2) {
    const size_t smem = bwd_readout_tc_smem_bytes();
    auto kernel = c2 ? wkv6_bwd_readout_tc_kernel<true, true> : wkv6_bwd_readout_tc_kernel<true, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)(B * H), kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], static_cast<const __nv_bfloat16*>(k), u,
        dS_T, nullptr, Q, nullptr, nullptr, dS_0, static_cast<__nv_bfloat16*>(dk), D, fallback, T,
        H, status, budget, 4000000000LL);
    return cudaGetLastError();
}

namespace {

// Decay gradient from the pair terms (the identity of csrc/backward.cu):
//     dlog w_t = E + sum_{s>t} P_s - sum_{s>=t} Q_s,   domega_t = dlog w_t (-exp(omega_t)),
// P and Q in token order.  First the column sums of P and of Q over each 64-token chunk (a
// launch each, queued right after the pass that writes the array, so that it runs beside
// the other pass), then per chunk the sums over the later chunks and a reverse scan over
// its own tokens.  One thread per channel and chunk, kDomegaChunks chunks of one (b,h) per
// CTA.  (One CTA per (b,h) walking its chunks backwards with a running total reads P and Q
// once instead of twice, but at 256 CTAs each chunk's loads wait in line: it measured
// slower.)
constexpr int kDomegaChunks = 4;

// sums[bh][n][64 * half + i] = sum over chunk n's tokens of X[t][i]
__global__ void __launch_bounds__(64 * kDomegaChunks)
wkv6_bwd_col_sums_kernel(const float* __restrict__ X, float* __restrict__ sums, int half, int T,
                         int H) {
    const int NC = (T + C - 1) / C, groups = (NC + kDomegaChunks - 1) / kDomegaChunks;
    const int g = blockIdx.x % groups, bh = blockIdx.x / groups, b = bh / H, h = bh - b * H;
    const int n = g * kDomegaChunks + (threadIdx.x >> 6), i = threadIdx.x & 63;
    if (n >= NC) return;
    const int t0 = n * C, valid = min(C, T - t0);
    const size_t stride = (size_t)H * 64, x0 = (((size_t)b * T + t0) * H + h) * 64 + i;
    // four partial sums: the loads of 8 tokens in flight, not one add chain
    float sx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int tt = 0; tt < valid; ++tt) sx[tt & 3] += X[x0 + tt * stride];
    sums[((size_t)bh * NC + n) * 128 + 64 * half + i] = (sx[0] + sx[1]) + (sx[2] + sx[3]);
}

// CTAs run from the last (b,h) to the first: the first of them find the P and Q the sums
// kernels read last still in L2.
__global__ void __launch_bounds__(64 * kDomegaChunks)
wkv6_bwd_domega_kernel(const float* __restrict__ P, const float* __restrict__ Q,
                       const float* __restrict__ Dw, const float* __restrict__ sums,
                       const float* __restrict__ E,
                       const __nv_bfloat16* __restrict__ omega, __nv_bfloat16* __restrict__ domega,
                       int T, int H) {
    const int NC = (T + C - 1) / C, groups = (NC + kDomegaChunks - 1) / kDomegaChunks;
    const int blk = gridDim.x - 1 - blockIdx.x;
    const int g = blk % groups, bh = blk / groups, b = bh / H, h = bh - b * H;
    const int n = g * kDomegaChunks + (threadIdx.x >> 6), i = threadIdx.x & 63;
    if (n >= NC) return;
    const int t0 = n * C, valid = min(C, T - t0);
    // E + sum over the later chunks of (P - Q), four independent partial sums
    const float* o = sums + (size_t)bh * NC * 128 + i;
    float part[4] = {E[(size_t)bh * 64 + i], 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int m = n + 1; m < NC; ++m) part[(m - n) & 3] += o[(size_t)m * 128] - o[(size_t)m * 128 + 64];
    float acc = (part[0] + part[1]) + (part[2] + part[3]);
    // reverse over this chunk: dlog w_t = acc_after(t) - Q_t, with acc_after(t) = E + sum_{s>t}
    // P_s - sum_{s>t} Q_s
    const size_t stride = (size_t)H * 64, x0 = (((size_t)b * T + t0) * H + h) * 64 + i;
#pragma unroll 8
    for (int tt = valid - 1; tt >= 0; --tt) {
        const size_t x = x0 + tt * stride;
        const float q = Q[x];
        const float dl = acc - q - (Dw != nullptr ? Dw[x] : 0.f);
        domega[x] = __float2bfloat16_rn(dl * -__expf(__bfloat162float(omega[x])));
        acc += P[x] - q;
    }
}

}  // namespace

cudaError_t launch_bwd_col_sums(const float* X, float* sums, int half, int B, int T, int H,
                                cudaStream_t st) {
    const long groups = ((T + C - 1) / C + kDomegaChunks - 1) / kDomegaChunks;
    const unsigned blocks = (unsigned)((long)B * H * groups);
    if (blocks == 0) return cudaSuccess;
    wkv6_bwd_col_sums_kernel<<<blocks, 64 * kDomegaChunks, 0, st>>>(X, sums, half, T, H);
    return cudaGetLastError();
}

cudaError_t launch_bwd_domega(const float* P, const float* Q, const float* D, const float* sums,
                              const float* E, const void* omega, void* domega, int B, int T,
                              int H, cudaStream_t st) {
    const long groups = ((T + C - 1) / C + kDomegaChunks - 1) / kDomegaChunks;
    const unsigned blocks = (unsigned)((long)B * H * groups);
    if (blocks == 0) return cudaSuccess;
    wkv6_bwd_domega_kernel<<<blocks, 64 * kDomegaChunks, 0, st>>>(P, Q, D, sums, E,
                                                  static_cast<const __nv_bfloat16*>(omega),
                                                  static_cast<__nv_bfloat16*>(domega), T, H);
    return cudaGetLastError();
}

}  // namespace goldwkv
