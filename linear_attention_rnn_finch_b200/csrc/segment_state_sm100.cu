// Segment states for the sequence split of the chunked prefill (sm_100a).
//
// A long sequence is cut into P segments that run on different SMs.  A segment p > 0 must
// start from the state left by the segments before it, which the recurrence of the
// GoldFinch review page (section 3.4, "Recurrent state update and output") fixes as
//     S_end = diag(G) S_start + sum_{t in segment} diag(prod_{t < tau in segment} w_tau) k_t^T v_t,
//     G = prod_{t in segment} w_t,
// i.e. an affine map of S_start.  This file computes, per segment, the local part
// S_loc (the sum, which is the segment's state from a zero start) and log2 G; the carry
// kernel then chains S_start(p+1) = diag(G_p) S_start(p) + S_loc(p).
//
// S_loc is built chunk by chunk with the suffix factorisation: inside a chunk,
//     Kt_s = k_s * 2^(sum_{s < tau < C} log2 w_tau)   (<= |k_s|: never overflows),
//     S <- diag(gamma) S + Kt^T V,  gamma = prod_{tau in chunk} w_tau,
// with the suffix sums accumulated directly (a sum of terms of one sign, not a difference
// of prefix sums), so any decay -- down to w = 0 -- is exact to fp32 rounding.  Kt is split
// into bf16 hi + lo parts; Kt^T V runs on tcgen05 as V^T (M=64) x Kt_hi + V^T x Kt_lo
// (N=64 each, accumulated in TMEM).
//
// Warp roles (320 threads, two CTAs per SM): warp 0 TMA (k, v, omega; 3-stage ring) and TMEM
// owner; warp 1 one MMA thread; warps 2-5 prep (16 tokens each); warps 6-9 the state update
// in registers, one warp per TMEM sub-partition.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "chunk_tiles.cuh"
#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

using namespace tiles;

constexpr int C = 64;
constexpr int kStages = 3;
constexpr int kPrepWarps = 4, kEpiWarps = 4;
constexpr int kTokPerWarp = C / kPrepWarps;   // 16
constexpr int kTmaWarp = 0, kMmaWarp = 1, kPrepWarp0 = 2, kEpiWarp0 = kPrepWarp0 + kPrepWarps;
constexpr int kPrepThreads = 32 * kPrepWarps, kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 32 * kPrepWarp0 + kPrepThreads + kEpiThreads;
constexpr uint32_t kTmemCols = 128;   // DU: 2 buffers x 64 columns (M = 64)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBarPrep = 1;
constexpr uint32_t IDESC_GU = ptx::idesc_bf16(64, 64, 1, 1);

struct __align__(1024) Smem {
    uint8_t in[kStages][3][kTile];   // k, v, omega tiles (TMA, 128B swizzle)
    uint8_t kt[2][2 * kTile];        // per parity: Kt_hi tile, then Kt_lo tile
    float qtot[2][kPrepWarps][64];   // per-warp sums of log2 w
    float gamma[2][64];
    uint64_t full[kStages], empty[kStages];
    uint64_t prep_done[2], op_free[2], ep_free[2], gu_done[2], du_free[2];
    uint32_t tmem_base;
    int abort;
    int stop_at;                     // no hand-over here: never <= a chunk index
};

// kC2: Finch-C2's normalised key k (1 - w) enters the state.
template <bool kC2>
__global__ void __launch_bounds__(kThreads, 2)
wkv6_segment_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_w, float* s_loc, float* log2g, int H,
                          int P, int seg_chunks, int* status, long long budget, long long drain_budget) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = smem_aligned<Smem>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // unit: segment pseg (< P-1, so every chunk is full) of sequence bh
    const int unit = blockIdx.x, nbh = gridDim.x / (P - 1);
    const int bh = unit % nbh, pseg = unit / nbh, b = bh / H, h = bh - (bh / H) * H;
    const int cseg = pseg * seg_chunks;
    const int NC = seg_chunks;
    const size_t out_idx = (size_t)bh * (P - 1) + pseg;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&s.full[i], 1);
            ptx::mbar_init(&s.empty[i], kPrepThreads + 1);   // prep reads k, omega; GU reads v
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.prep_done[i], kPrepThreads);
            ptx::mbar_init(&s.op_free[i], 1);
            ptx::mbar_init(&s.ep_free[i], kEpiThreads);
            ptx::mbar_init(&s.gu_done[i], 1);
            ptx::mbar_init(&s.du_free[i], kEpiThreads);
        }
        ptx::fence_mbar_init();
        s.abort = 0;
        s.stop_at = 0x7fffffff;
    }
    if (warp == kTmaWarp) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_k);
            ptx::prefetch_tensormap(&tm_v);
            ptx::prefetch_tensormap(&tm_w);
            int last[kStages] = {-1, -1, -1};
            for (int n = 0; n < NC; ++n) {
                const int st = n % kStages;
                if (n >= kStages && !wait_soft(s, &s.empty[st], (uint32_t)((n / kStages - 1) & 1), budget)) break;
                // every chunk of a segment before the last is inside the sequence
                if (!gw_check(status, pseg < P - 1 && h < H && b < nbh / H)) break;
                ptx::mbar_arrive_expect_tx(&s.full[st], 3 * kTile);
                ptx::tma_load_4d(s.in[st][0], &tm_k, &s.full[st], 0, h, (cseg + n) * C, b);
                ptx::tma_load_4d(s.in[st][1], &tm_v, &s.full[st], 0, h, (cseg + n) * C, b);
                ptx::tma_load_4d(s.in[st][2], &tm_w, &s.full[st], 0, h, (cseg + n) * C, b);
                last[st] = n;
            }
            for (int st = 0; st < kStages; ++st)
                if (last[st] >= 0)
                    ptx::mbar_wait(&s.full[st], (uint32_t)((last[st] / kStages) & 1), drain_budget);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ GU issue
        if (lane == 0) {
            int last = -1;
            for (int n = 0; n < NC; ++n) {
                const int pb = n & 1, st = n % kStages;
                if (!wait_soft(s, &s.prep_done[pb], (uint32_t)((n >> 1) & 1), budget)) break;
                if (n >= 2 && !wait_soft(s, &s.du_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget)) break;
                ptx::tc_fence_after();
                const uint32_t v_tile = ptx::smem_addr(s.in[st][1]);
                const uint32_t kt = ptx::smem_addr(s.kt[pb]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // DU = V^T x Kt_hi + V^T x Kt_lo
                    ptx::mma_bf16(tmem + 64 * pb, ptx::desc_mnmajor(v_tile + 2048 * kq),
                                  ptx::desc_mnmajor(kt + 2048 * kq), IDESC_GU, kq > 0);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    ptx::mma_bf16(tmem + 64 * pb, ptx::desc_mnmajor(v_tile + 2048 * kq),
                                  ptx::desc_mnmajor(kt + kTile + 2048 * kq), IDESC_GU, 1);
                ptx::mma_commit(&s.gu_done[pb]);
                ptx::mma_commit(&s.op_free[pb]);
                ptx::mma_commit(&s.empty[st]);
                last = n;
            }
            if (last >= 0) ptx::mbar_wait(&s.gu_done[last & 1], (uint32_t)((last >> 1) & 1), drain_budget);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ prep (4 warps)
        // warp g: tokens 16g .. 16g+15; lane = channel pair (2l, 2l+1); log2 units
        const int g = warp - kPrepWarp0;
        const int c2 = 2 * lane;
        const int chunk = lane >> 2;
        const uint32_t cbyte = (uint32_t)(lane & 3) * 4;
        const float2 l2e = make_float2(kLog2e, kLog2e);
        float2 lg = make_float2(0.f, 0.f);   // -sum of log2 w over the segment (warp 0)
        for (int n = 0; n < NC; ++n) {
            const int pb = n & 1, st = n % kStages;
            bool ok = wait_soft(s, &s.full[st], (uint32_t)((n / kStages) & 1), budget);
            if (n >= 2) {
                ok = ok && wait_soft(s, &s.op_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget);
                ok = ok && wait_soft(s, &s.ep_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget);
            }
            if (named_bar_any(kBarPrep, kPrepThreads, !ok || ld_volatile(&s.abort))) break;
            const uint8_t* k_tile = s.in[st][0];
            const uint8_t* w_tile = s.in[st][2];
            // -log2 w = exp(omega) log2(e); exclusive suffix sums inside the warp's tokens,
            // accumulated from the last token down (terms of one sign)
            float2 suf[kTokPerWarp];
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = kTokPerWarp - 1; q >= 0; --q) {
                const float2 om = __fmul2_rn(unpack2(lds32(w_tile, sw_off(kTokPerWarp * g + q, chunk) + cbyte)), l2e);
                suf[q] = acc;
                acc = __ffma2_rn(make_float2(fast_exp2(om.x), fast_exp2(om.y)), l2e, acc);
            }
            *reinterpret_cast<float2*>(&s.qtot[pb][g][c2]) = acc;   // -sum of the warp's log2 w
            named_bar(kBarPrep, kPrepThreads);
            float2 after = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kPrepWarps; ++w) {
                const float2 qv = *reinterpret_cast<const float2*>(&s.qtot[pb][w][c2]);
                if (w > g) after = __fadd2_rn(after, qv);
                tot = __fadd2_rn(tot, qv);
            }
            uint8_t* kt_hi = s.kt[pb];
            uint8_t* kt_lo = s.kt[pb] + kTile;
#pragma unroll
            for (int q = 0; q < kTokPerWarp; ++q) {
                const uint32_t o = sw_off(kTokPerWarp * g + q, chunk) + cbyte;
                const float2 x = __fadd2_rn(after, suf[q]);          // >= 0
                float2 f = make_float2(fast_exp2(-x.x), fast_exp2(-x.y));
                if (kC2) {   // times 1 - w = 1 - exp(-exp(omega)) of this token
                    const float2 om = __fmul2_rn(unpack2(lds32(w_tile, o)), l2e);
                    f = __fmul2_rn(f, one_minus_exp_neg2(make_float2(fast_exp2(om.x), fast_exp2(om.y))));
                }
                uint32_t hi, lo;
                split2(__fmul2_rn(unpack2(lds32(k_tile, o)), f), hi, lo);
                sts32(kt_hi, o, hi);
                sts32(kt_lo, o, lo);
            }
            mbar_arrive(&s.empty[st]);       // k and omega of this stage read
            if (g == 0) {
                *reinterpret_cast<float2*>(&s.gamma[pb][c2]) = make_float2(fast_exp2(-tot.x), fast_exp2(-tot.y));
                lg = __fadd2_rn(lg, tot);
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.prep_done[pb]);
        }
        if (g == 0 && !ld_volatile(&s.abort))
            *reinterpret_cast<float2*>(log2g + out_idx * 64 + c2) = make_float2(-lg.x, -lg.y);
    } else {
        // ------------------------------------------------------------ state (4 warps)
        // warp q = warp % 4 (its TMEM sub-partition): rows j = 16q + l/4 and +8 of S^T,
        // columns i = 32h + 8k + 2(l%4) + {0,1} for column halves h = 0, 1
        const int q = warp & 3;
        const int r0 = 16 * q + (lane >> 2), r1 = r0 + 8;
        const int cl = 2 * (lane & 3);
        const uint32_t lane_h0 = (uint32_t)(32 * q) << 16;
        float2 S0[8], S1[8];   // index 4h + k
#pragma unroll
        for (int k = 0; k < 8; ++k) S0[k] = S1[k] = make_float2(0.f, 0.f);
        int n = 0;
        for (; n < NC; ++n) {
            const int pb = n & 1;
            // DU of chunk n; gamma of chunk n reaches us from prep through prep_done -> the MMA
            // thread's acquire -> its commit on gu_done
            if (!wait_soft(s, &s.gu_done[pb], (uint32_t)((n >> 1) & 1), budget))
                break;   // abort: every later wait returns at once as well
            ptx::tc_fence_after();
            uint32_t ua[16], ub[16];
            tmem_ld16x4(tmem + lane_h0 + 64 * pb, ua);
            tmem_ld16x4(tmem + lane_h0 + 64 * pb + 32, ub);
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            mbar_arrive(&s.du_free[pb]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 g0 = *reinterpret_cast<const float2*>(&s.gamma[pb][cl + 8 * k]);
                const float2 g1 = *reinterpret_cast<const float2*>(&s.gamma[pb][32 + cl + 8 * k]);
                S0[k] = __ffma2_rn(g0, S0[k], lo_pair(ua, k));
                S1[k] = __ffma2_rn(g0, S1[k], hi_pair(ua, k));
                S0[4 + k] = __ffma2_rn(g1, S0[4 + k], lo_pair(ub, k));
                S1[4 + k] = __ffma2_rn(g1, S1[4 + k], hi_pair(ub, k));
            }
            mbar_arrive(&s.ep_free[pb]);
        }
        if (n == NC && !ld_volatile(&s.abort)) {
            float* dst = s_loc + out_idx * 4096;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = 32 * (k >> 2) + cl + 8 * (k & 3);
                dst[i * 64 + r0] = S0[k].x;
                dst[(i + 1) * 64 + r0] = S0[k].y;
                dst[i * 64 + r1] = S1[k].x;
                dst[(i + 1) * 64 + r1] = S1[k].y;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (s.abort && tid == 0) atomicExch(status, 1);
    if (warp == kTmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// One CTA per (b,h), 256 threads, 16 state elements each (row i = tid / 4, 16 columns).
__global__ void __launch_bounds__(256)
wkv6_segment_carry_kernel(const float* state_in, const float* s_loc, const float* log2g,
                          float* s_mid, int P) {
    const int bh = blockIdx.x, i = threadIdx.x >> 2, j0 = 16 * (threadIdx.x & 3);
    float S[16];
    const float* src = state_in ? state_in + (size_t)bh * 4096 + i * 64 + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float4 x = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    for (int p = 0; p < P - 1; ++p) {
        const size_t idx = (size_t)bh * (P - 1) + p;
        const float gi = exp2f(log2g[idx * 64 + i]);
        const float* loc = s_loc + idx * 4096 + i * 64 + j0;
        float* out = s_mid + idx * 4096 + i * 64 + j0;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            const float4 l = *reinterpret_cast<const float4*>(loc + j);
            S[j] = fmaf(gi, S[j], l.x);
            S[j + 1] = fmaf(gi, S[j + 1], l.y);
            S[j + 2] = fmaf(gi, S[j + 2], l.z);
            S[j + 3] = fmaf(gi, S[j + 3], l.w);
            *reinterpret_cast<float4*>(out + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
}

// States entering P consecutive segments given each one's local state and log2 decay, laid
// out segment-major ([p][bh]): s_in[0] = state0 (zero if null), s_in[p+1] = 2^g[p] (rows)
// s_in[p] + s_loc[p], p = 0 .. P-1 (s_in has P + 1 entries).  One CTA per (b,h), a thread
// per row i and 16 columns.
__global__ void __launch_bounds__(256)
wkv6_segment_carry_ranks_kernel(const float* state0, const float* s_loc, const float* log2g,
                                float* s_in, int P, int nbh) {
    const int bh = blockIdx.x, i = threadIdx.x >> 2, j0 = 16 * (threadIdx.x & 3);
    float S[16];
    const float* src = state0 ? state0 + (size_t)bh * 4096 + i * 64 + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float4 x = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    for (int p = 0; p <= P; ++p) {
        float* out = s_in + ((size_t)p * nbh + bh) * 4096 + i * 64 + j0;
#pragma unroll
        for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(out + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        if (p == P) break;
        const size_t idx = (size_t)p * nbh + bh;
        const float gi = exp2f(log2g[idx * 64 + i]);
        const float* loc = s_loc + idx * 4096 + i * 64 + j0;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            const float4 l = *reinterpret_cast<const float4*>(loc + j);
            S[j] = fmaf(gi, S[j], l.x);
            S[j + 1] = fmaf(gi, S[j + 1], l.y);
            S[j + 2] = fmaf(gi, S[j + 2], l.z);
            S[j + 3] = fmaf(gi, S[j + 3], l.w);
        }
    }
}

}  // namespace

cudaError_t launch_segment_carry_ranks(const float* state0, const float* s_loc,
                                       const float* log2g, float* s_in, int B, int H, int P,
                                       cudaStream_t st) {
    if (B * H == 0) return cudaSuccess;
    wkv6_segment_carry_ranks_kernel<<<(unsigned)(B * H), 256, 0, st>>>(state0, s_loc, log2g, s_in,
                                                                      P, B * H);
    return cudaGetLastError();
}

size_t segment_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_segment_states(const CUtensorMap* maps, float* s_loc, float* log2g, int B,
                                  int T, int H, Segments seg, Variant var, int* status,
                                  long long budget, cudaStream_t st) {
    (void)T;
    if (seg.P < 2) return cudaSuccess;
    const size_t smem = segment_smem_bytes();
    auto kernel = var.uprime ? wkv6_segment_state_kernel<true> : wkv6_segment_state_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)(B * H * (seg.P - 1)), kThreads, smem, st>>>(
        maps[1], maps[2], maps[3], s_loc, log2g, H, seg.P, seg.seg_chunks, status, budget,
        4000000000LL);
    return cudaGetLastError();
}

cudaError_t launch_segment_carry(const float* state_in, const float* s_loc, const float* log2g,
                                 float* s_mid, int B, int H, int P, cudaStream_t st) {
    if (P < 2) return cudaSuccess;
    wkv6_segment_carry_kernel<<<(unsigned)(B * H), 256, 0, st>>>(state_in, s_loc, log2g, s_mid, P);
    return cudaGetLastError();
}

}  // namespace goldwkv
