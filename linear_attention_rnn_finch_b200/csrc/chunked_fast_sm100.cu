// Chunked WKV6 prefill, fast path: warp-specialised tcgen05 pipeline (sm_100a).
//
// Same recurrence as chunked_sm100.cu (GoldFinch review page, section 3.4: decay
// w = exp(-exp(omega)), state S_t = diag(w_t) S_{t-1} + k_t^T v_t, readout
// y_t = r_t . (diag(u) k_t^T v_t + S_{t-1})), for chunks whose decay range is moderate.
//
// One-sided factorisation.  Let L_t = sum_{tau<=t} log w_tau inside a chunk of C = 64
// tokens (L <= 0, decreasing).  If every channel's total L_{C-1} >= -kMaxLogRange, the
// intra-chunk factor prod_{s<tau<t} w = exp(L_{t-1} - L_s) splits as
//     exp(L_{t-1}) * exp(-L_s)  with  exp(L_{t-1}) in (0, 1],  exp(-L_s) in [1, e^60],
// both representable in bf16 / fp32 without overflow, so
//     Rt_t = r_t * exp(L_{t-1}),  Kh_s = k_s * exp(-L_s)
//     y_t  = Rt_t . S + sum_{s<t} (Rt_t . Kh_s) v_s + (r_t . (u * k_t)) v_t
//     S'   = diag(gamma) (S + Kh^T V),  gamma = exp(L_{C-1}).
// A chunk that fails the test stops this kernel for its (b,h): the state S entering that
// chunk and the chunk index are handed (through the workspace) to the level-factorised
// kernel, which finishes the sequence.  Nothing is clamped.
//
// Precision.  Rt, S and A are split into hi = bf16(x) and lo = bf16(x - hi), and Kh is
// split for the state increment.  Where both parts of the A operand meet the same B operand
// they are stacked into M = 128 (rows 0-7 of every 16-row group hold hi parts of 8 tokens,
// rows 8-15 the lo parts of the same tokens), and a 16x256b TMEM load hands each thread the
// hi and lo element of the same (token, column), so the combination is one add in
// registers.  Where the split operand is B (Kh in the increment, S in the readout), its two
// parts are side by side in N, and the epilogue adds the two column blocks (one tcgen05.mma
// of N = 128 costs the tensor pipe about as long as one of N = 64).
//
// Products per chunk n (bf16 operands, fp32 accumulators in TMEM):
//   GU(n): V^T (M=64) x [Kh_hi | Kh_lo] (N=128) -> DU = (Kh^T V)^T, the state increment,
//          which depends only on the chunk's own operands;
//   SC(n): [Rt_hi ; Rt_lo] (M=128) x Kh_hi^T (N=64)             intra-chunk scores;
//   RO(n): [Rt_hi ; Rt_lo] x [S_hi^T ; S_lo^T] (N=128)          readout of S_{n-1} -> Y;
//   GA(n): [A_hi ; A_lo] x V (N=64), accumulated into Y's first 64 columns
//                                                               A = masked scores + bonus.
//
// Roles (16 warps, no dedicated producer or issuer warps: a thread that has just finished
// a step, or is between two steps of its own work, issues the copies and products that
// follow, so no warp does nothing but poll):
//   warps 0-7, prep: two groups of 4 warps taking alternate chunks (group g: n = g mod 2).
//     A warp takes 16 tokens; a thread takes 8 channels (one 16-byte column of the tile) of
//     4 consecutive tokens: exp(omega), the log-decay prefix (serial over its 4 tokens, a
//     shuffle scan over the warp's 4 runs, a shared-memory sum over the group's warps), the
//     range test, Rt / Kh hi/lo with 16-byte stores, the bonus (shuffle-reduced over the 8
//     channel columns) and gamma.  Lane 0 of three of the group's warps issues tensor-core
//     work, so that one issuer's wait on the tensor pipe does not hold up the others:
//       warp 0, after chunk n: the r / k / omega copy of chunk n+3, GU(n) and SC(n);
//       warp 1, after chunk n: GA(n-1) (the other group's chunk), once the epilogue stored
//               A(n-1) and RO(n-1) is complete;
//       warp 2, between the two passes of chunk n: RO(n-2), once the epilogue stored S_{n-3}
//               (before pass 2 rewrites the Rt buffer RO(n-2) reads).
//   warps 8-15, epilogue, per chunk n: state(n) = gamma (S + DU); S_n hi/lo for RO(n+1);
//     A(n); the output of chunk n-1 (Y -> y); its elected thread loads v of chunk n+3.
//     The epilogue issues no tensor-core work.
// The fp32 state stays in the epilogue's registers.  Handshakes are mbarriers (tensor-core
// commits, copy completion, epilogue arrivals) and named barriers inside a group; every
// mbarrier wait is bounded.  A barrier phase is never completed while a waiter may still be
// waiting for the phase before it (its parity wait would alias): commits follow from the
// data dependencies, and a hand-over or give-up that could break that order skips its
// commit or waits first.
#include <cuda.h>
#include <cuda_bf16.h>
#include <limits.h>

#include "common.cuh"
#include "internal.h"
#include "chunk_tiles.cuh"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

using namespace tiles;

constexpr int C = 64;
constexpr int kStagesRkw = 3, kStagesV = 4;
constexpr int kPrepGroups = 2, kGroupWarps = 4, kEpiWarps = 8;
constexpr int kPrepWarps = kPrepGroups * kGroupWarps;
constexpr int kEpiWarp0 = kPrepWarps;
constexpr int kGroupThreads = 32 * kGroupWarps, kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 32 * (kPrepWarps + kEpiWarps);
constexpr int kEpiLeader = 32 * kEpiWarp0;   // the epilogue's issuing thread
// an epilogue thread covers 4 column pairs (one 32-column half) of each accumulator
constexpr int kPairs = 4;
constexpr uint32_t kTmemCols = 512;
// DU: 1 buffer x 128 columns (M=64; Kh_hi part, then Kh_lo part); SC: 2 x 64 (M=128); Y: 2 x 128
// (M=128; the S_hi part, with GA accumulated onto it, then the S_lo part)
constexpr uint32_t COL_DU = 0, COL_SC = 128, COL_Y = 256;
// log2 of the largest factor exp(-L_s) allowed: ln range 60 -> log2 range 86.56
constexpr float kMaxLog2Range = 86.5617f;
constexpr float kLog2e = 1.4426950408889634f;
// named barriers (id 0 is __syncthreads): one per prep group, one for the epilogue, and one
// per pair of epilogue warps that hold the two column halves of the same rows (GroupNorm)
constexpr int kBarPrep0 = 1, kBarEpi = kBarPrep0 + kPrepGroups, kBarPair0 = kBarEpi + 1;
constexpr int kNoStop = INT_MAX;

constexpr uint32_t IDESC_GU = ptx::idesc_bf16(64, 128, 1, 1);
constexpr uint32_t IDESC_SC = ptx::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_RO = ptx::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t IDESC_GA = ptx::idesc_bf16(128, 64, 0, 1);

struct __align__(1024) Smem {
    uint8_t rkw[kStagesRkw][3][kTile];  // r, k, omega tiles (TMA, 128B swizzle); chunk n in n % 3
    uint8_t vt[kStagesV][kTile];        // v tiles; chunk n in n % 4
    uint8_t rt[2][2 * kTile];           // per parity: Rt hi/lo, 128 stacked rows
    uint8_t kh[2][2 * kTile];           // per parity: Kh_hi tile, then Kh_lo tile
    uint8_t sb[2][2 * kTile];           // S_hi^T tile, then S_lo^T tile; sb[m & 1] feeds RO(m)
    uint8_t at[2 * kTile];              // A hi/lo, 128 stacked rows
    // prep: per-warp sums of log2 w, 8 channels per 16-byte pair of columns, rows padded to
    // 12 floats so that the 8 column groups a quarter-warp reads fall in distinct banks
    float qtot[kPrepGroups][kGroupWarps][8][12];
    float gamma[4][64];                 // gamma and bonus of chunk n in slot n % 4
    float bonus[4][64];
    uint64_t full_rkw[kStagesRkw], full_v[kStagesV];
    // prep issuers' commits for chunk n in slot n & 1: mm_done after GU(n) + SC(n), op_free
    // after RO(n), ya_done after GA(n); drain[g][i]: issuer i of group g's last commit
    uint64_t mm_done[2], op_free[2], ya_done[2], drain[kPrepGroups][3];
    // epilogue arrivals: du_free (DU read), ep_free[n % 4] (gamma / bonus of n read),
    // a_ready[n & 1] (A(n) stored, SC(n) read), s_ready[n & 1] (S_{n-1} stored in sb[n & 1]
    // and Y[n & 1] free: RO(n) may run)
    uint64_t du_free, ep_free[4], a_ready[2], s_ready[2];
    int last_rkw[kStagesRkw], last_v[kStagesV];    // latest chunk loaded into each stage
    uint32_t tmem_base;
    int abort;
    int stop_at;                        // first chunk handed to the level kernel (kNoStop: none)
    // GroupNorm output stage: the head's gamma / beta, and per output-chunk parity the
    // (mean, M2) of each row's two 32-column halves
    float gn_gamma[64], gn_beta[64];
    float2 gn_mom[2][2][64];
};

__device__ __forceinline__ void sts128(uint8_t* base, uint32_t off, uint32_t a, uint32_t b,
                                       uint32_t c, uint32_t d) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(a, b, c, d);
}
// 16-byte shared-memory load issued where it stands (next to its use), which bounds the
// registers the unrolled token loop keeps live.
__device__ __forceinline__ uint4 lds128v(const uint8_t* base, uint32_t off) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(ptx::smem_addr(base + off)));
    return v;
}
// word q (0..3) of a 16-byte vector; q is a compile-time constant after unrolling
__device__ __forceinline__ uint32_t word(const uint4& v, int q) {
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
__device__ __forceinline__ float2 shfl_up2(float2 v, int d) {
    return make_float2(__shfl_up_sync(0xffffffffu, v.x, d), __shfl_up_sync(0xffffffffu, v.y, d));
}
__device__ __forceinline__ float2 exp2_2(float2 x) {
    return make_float2(fast_exp2(x.x), fast_exp2(x.y));
}
// stop reading / producing chunk n: the CTA aborted, or this (b,h) was handed over at or
// before n
__device__ __forceinline__ bool stopped_at(const Smem& s, int n) {
    return ld_volatile(&s.abort) != 0 || ld_volatile(&s.stop_at) <= n;
}

// (mean, M2) of the 8 values of a thread's 4 column pairs (two passes over the registers)
__device__ __forceinline__ float2 moments8(const float2 (&v)[kPairs]) {
    float sm = 0.f;
#pragma unroll
    for (int j = 0; j < kPairs; ++j) sm += v[j].x + v[j].y;
    const float mean = sm * 0.125f;
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        const float d0 = v[j].x - mean, d1 = v[j].y - mean;
        q = fmaf(d0, d0, fmaf(d1, d1, q));
    }
    return make_float2(mean, q);
}
// (mean, M2) of the union of two disjoint sets of n values each (Chan et al.'s update with
// n_a = n_b = n: mean = (mean_a + mean_b) / 2, M2 = M2_a + M2_b + (mean_b - mean_a)^2 n / 2)
__device__ __forceinline__ float2 merge_equal(float2 a, float2 b, float n) {
    const float d = b.x - a.x;
    return make_float2(0.5f * (a.x + b.x), a.y + b.y + 0.5f * n * d * d);
}
__device__ __forceinline__ float2 shfl_xor2(float2 v, int o) {
    return make_float2(__shfl_xor_sync(0xffffffffu, v.x, o), __shfl_xor_sync(0xffffffffu, v.y, o));
}

// Output of chunk m (plus the second value u' of Finch-C2, whose words up0 / up1 for rows
// r0 / r1 the caller loaded ahead of time): y = the hi and lo rows of both column blocks of
// Y[m & 1], stored as bf16
// (or fp32 rows to y_raw).  The caller has waited for GA(m).  col0: first column of this
// thread's pairs (pair j at col0 + 8j).
template <bool kC2, bool kGN>
__device__ __forceinline__ void output_chunk(Smem& s, float gn_eps, int m, int c0, uint32_t tmem, uint32_t lane_h0,
                                             uint32_t lane_h1, int col0, int cl, int r0, int r1,
                                             int b, int h, int T, int H, __nv_bfloat16* y,
                                             float* y_raw, const uint32_t (&up0)[kPairs],
                                             const uint32_t (&up1)[kPairs]) {
    const int yb = m & 1;
    float2 Y0[kPairs], Y1[kPairs];
    {
        uint32_t a[16], c[16], a2[16], c2[16];
        tmem_ld16x4(tmem + lane_h0 + COL_Y + 128 * yb + col0, a);
        tmem_ld16x4(tmem + lane_h1 + COL_Y + 128 * yb + col0, c);
        tmem_ld16x4(tmem + lane_h0 + COL_Y + 128 * yb + 64 + col0, a2);
        tmem_ld16x4(tmem + lane_h1 + COL_Y + 128 * yb + 64 + col0, c2);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kPairs; ++j) {
            Y0[j] = __fadd2_rn(rows_sum(a, j), rows_sum(a2, j));
            Y1[j] = __fadd2_rn(rows_sum(c, j), rows_sum(c2, j));
        }
    }
    ptx::tc_fence_before();
    const int tc = (c0 + m) * C;
    const int valid = min(C, T - tc);
    const size_t row0 = ((size_t)b * T + (size_t)tc + r0) * H + h;
    const size_t row1 = ((size_t)b * T + (size_t)tc + r1) * H + h;
    if (kGN) {
        // base Finch's output stage: GroupNorm of each (token, head) row of 64 channels, the
        // head's affine, times the gate (words up0 / up1, loaded beforehand).  Mean and M2 of
        // this thread's 8 values, merged over the 4 lanes of its 32-column half, then with
        // the other half's (the partner warp, through shared memory)
        const int half = col0 >> 5, slot = m & 1;
        float2 mo0 = moments8(Y0), mo1 = moments8(Y1);   // (mean, M2) over 8 values
        mo0 = merge_equal(mo0, shfl_xor2(mo0, 1), 8.f);   // 16 values
        mo1 = merge_equal(mo1, shfl_xor2(mo1, 1), 8.f);
        mo0 = merge_equal(mo0, shfl_xor2(mo0, 2), 16.f);  // 32: the half
        mo1 = merge_equal(mo1, shfl_xor2(mo1, 2), 16.f);
        if (cl == 0) {
            s.gn_mom[slot][half][r0] = mo0;
            s.gn_mom[slot][half][r1] = mo1;
        }
        named_bar(kBarPair0 + ((r0 >> 4) & 3), 64);
        mo0 = merge_equal(mo0, s.gn_mom[slot][half ^ 1][r0], 32.f);   // 64: the row
        mo1 = merge_equal(mo1, s.gn_mom[slot][half ^ 1][r1], 32.f);
        const float inv0 = rsqrtf(mo0.y * (1.f / 64.f) + gn_eps);
        const float inv1 = rsqrtf(mo1.y * (1.f / 64.f) + gn_eps);
#pragma unroll
        for (int jj = 0; jj < kPairs; ++jj) {
            const int j = col0 + 8 * jj + cl;
            const float2 g = *reinterpret_cast<const float2*>(&s.gn_gamma[j]);
            const float2 be = *reinterpret_cast<const float2*>(&s.gn_beta[j]);
            const float2 gt0 = unpack2(up0[jj]), gt1 = unpack2(up1[jj]);
            const float2 a0 = make_float2(fmaf((Y0[jj].x - mo0.x) * inv0, g.x, be.x) * gt0.x,
                                          fmaf((Y0[jj].y - mo0.x) * inv0, g.y, be.y) * gt0.y);
            const float2 a1 = make_float2(fmaf((Y1[jj].x - mo1.x) * inv1, g.x, be.x) * gt1.x,
                                          fmaf((Y1[jj].y - mo1.x) * inv1, g.y, be.y) * gt1.y);
            if (r0 < valid) *reinterpret_cast<uint32_t*>(y + row0 * 64 + j) = pack2(a0.x, a0.y);
            if (r1 < valid) *reinterpret_cast<uint32_t*>(y + row1 * 64 + j) = pack2(a1.x, a1.y);
        }
        return;
    }
#pragma unroll
    for (int jj = 0; jj < kPairs; ++jj) {
        const int j = col0 + 8 * jj + cl;
        if (kC2) {   // Finch-C2: the second value u'_t joins the readout (loaded beforehand)
            Y0[jj] = __fadd2_rn(Y0[jj], unpack2(up0[jj]));
            Y1[jj] = __fadd2_rn(Y1[jj], unpack2(up1[jj]));
        }
        if (y_raw != nullptr) {
            if (r0 < valid) *reinterpret_cast<float2*>(y_raw + row0 * 64 + j) = Y0[jj];
            if (r1 < valid) *reinterpret_cast<float2*>(y_raw + row1 * 64 + j) = Y1[jj];
        } else {
            if (r0 < valid) *reinterpret_cast<uint32_t*>(y + row0 * 64 + j) = pack2(Y0[jj].x, Y0[jj].y);
            if (r1 < valid) *reinterpret_cast<uint32_t*>(y + row1 * 64 + j) = pack2(Y1[jj].x, Y1[jj].y);
        }
    }
}

// Words of a [B][T][H][64] bf16 tensor (u' of Finch-C2, or the GroupNorm gate) for chunk
// (c0 + m), this thread's rows r0, r1 and its column pairs; rows past T read as zero, and a
// null tensor as bf16 ones.  Issued well before output_chunk needs them.
__device__ __forceinline__ void load_uprime(const __nv_bfloat16* __restrict__ uprime, int m, int c0,
                                            int b, int h, int T, int H, int col0, int cl, int r0, int r1,
                                            uint32_t (&up0)[kPairs], uint32_t (&up1)[kPairs]) {
    const int tc = (c0 + m) * C;
    const int valid = min(C, T - tc);
    const size_t row0 = ((size_t)b * T + (size_t)tc + r0) * H + h;
    const size_t row1 = ((size_t)b * T + (size_t)tc + r1) * H + h;
    constexpr uint32_t kOnes = 0x3F803F80u;   // two bf16 1.0
#pragma unroll
    for (int jj = 0; jj < kPairs; ++jj) {
        const int j = col0 + 8 * jj + cl;
        if (uprime == nullptr) {
            up0[jj] = up1[jj] = kOnes;
            continue;
        }
        up0[jj] = r0 < valid ? __ldg(reinterpret_cast<const unsigned int*>(uprime + row0 * 64 + j)) : 0u;
        up1[jj] = r1 < valid ? __ldg(reinterpret_cast<const unsigned int*>(uprime + row1 * 64 + j)) : 0u;
    }
}

// S_hi^T at tile, S_lo^T at tile + kTile: this thread's rows j = r0, r1, its column pairs i
// in 16-byte column chunks q0 .. q0 + 3
__device__ __forceinline__ void store_state(uint8_t* tile, const float2 (&S0)[kPairs],
                                            const float2 (&S1)[kPairs], int r0, int r1, int q0,
                                            uint32_t cb) {
#pragma unroll
    for (int k = 0; k < kPairs; ++k) {
        uint32_t hi, lo;
        split2(S0[k], hi, lo);
        sts32(tile, sw_off(r0, q0 + k) + cb, hi);
        sts32(tile + kTile, sw_off(r0, q0 + k) + cb, lo);
        split2(S1[k], hi, lo);
        sts32(tile, sw_off(r1, q0 + k) + cb, hi);
        sts32(tile + kTile, sw_off(r1, q0 + k) + cb, lo);
    }
}

// The CTA's unit and the bounds its copies must stay in (checked in debug builds only).
struct Unit {
    int h, b, cseg, NC, T, H, B;
    int* status;
};
// chunk n of the unit is a valid copy source: in the segment, the sequence and the tensor
__device__ __forceinline__ bool copy_ok(const Unit& u, int n) {
    return gw_check(u.status, n >= 0 && n < u.NC && (u.cseg + n) * C < u.T && u.h >= 0 &&
                                  u.h < u.H && u.b >= 0 && u.b < u.B);
}

// r, k, omega tiles of chunk n into stage n % 3 (one thread)
__device__ __forceinline__ void load_rkw(Smem& s, const CUtensorMap* tm_r, const CUtensorMap* tm_k,
                                         const CUtensorMap* tm_w, int n, const Unit& u) {
    if (!copy_ok(u, n)) return;
    const int st = n % kStagesRkw, cseg = u.cseg, h = u.h, b = u.b;
    ptx::mbar_arrive_expect_tx(&s.full_rkw[st], 3 * kTile);
    ptx::tma_load_4d(s.rkw[st][0], tm_r, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
    ptx::tma_load_4d(s.rkw[st][1], tm_k, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
    ptx::tma_load_4d(s.rkw[st][2], tm_w, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
    s.last_rkw[st] = n;
}
// v tile of chunk n into stage n % 4 (one thread)
__device__ __forceinline__ void load_v(Smem& s, const CUtensorMap* tm_v, int n, const Unit& u) {
    if (!copy_ok(u, n)) return;
    const int st = n % kStagesV, cseg = u.cseg, h = u.h, b = u.b;
    ptx::mbar_arrive_expect_tx(&s.full_v[st], kTile);
    ptx::tma_load_4d(s.vt[st], tm_v, &s.full_v[st], 0, h, (cseg + n) * C, b);
    s.last_v[st] = n;
}

// kC2: Finch-C2 exact form -- key k (1 - w), no static bonus, second value uprime added.
// kGN: base form with the GroupNorm + gate output stage (gn).
// kQ: no bonus, query r (1 - w) (Variant::query_c2).
template <bool kC2, bool kGN, bool kQ>
__global__ void __launch_bounds__(kThreads, 1)
wkv6_fast_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                 const float* __restrict__ u, const float* s_in, float* s_out,
                 __nv_bfloat16* __restrict__ y, float* __restrict__ y_raw,
                 const __nv_bfloat16* __restrict__ uprime, const GnOut gn, int T, int H,
                 Segments seg, int* status, int* handoff_chunk, float* handoff_state,
                 long long budget, long long drain_budget) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = smem_aligned<Smem>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // unit: segment pseg of sequence bh; chunks cseg .. cseg + NC - 1 (absolute indices)
    const int unit = blockIdx.x, nbh = gridDim.x / seg.P;
    const int bh = unit % nbh, pseg = unit / nbh, b = bh / H, h = bh - (bh / H) * H;
    const int cseg = pseg * seg.seg_chunks;
    const int NC = min((T + C - 1) / C, cseg + seg.seg_chunks) - cseg;
    const Unit cu{h, b, cseg, NC, T, H, nbh / H, status};

    if (tid == 0) {
        for (int i = 0; i < kStagesRkw; ++i) {
            ptx::mbar_init(&s.full_rkw[i], 1);
            s.last_rkw[i] = -1;
        }
        for (int i = 0; i < kStagesV; ++i) {
            ptx::mbar_init(&s.full_v[i], 1);
            s.last_v[i] = -1;
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.mm_done[i], 1);
            ptx::mbar_init(&s.op_free[i], 1);
            ptx::mbar_init(&s.ya_done[i], 1);
            ptx::mbar_init(&s.a_ready[i], kEpiThreads);
            ptx::mbar_init(&s.s_ready[i], kEpiThreads);
        }
        for (int i = 0; i < kPrepGroups; ++i)
            for (int j = 0; j < 3; ++j) ptx::mbar_init(&s.drain[i][j], 1);
        ptx::mbar_init(&s.du_free, kEpiThreads);
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&s.ep_free[i], kEpiThreads);
        ptx::fence_mbar_init();
        s.abort = 0;
        s.stop_at = kNoStop;
        ptx::prefetch_tensormap(&tm_r);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_w);
        // the first chunks' copies; later ones are issued as stages are released
        for (int n = 0; n < min(NC, kStagesRkw); ++n) load_rkw(s, &tm_r, &tm_k, &tm_w, n, cu);
        for (int n = 0; n < min(NC, kStagesV); ++n) load_v(s, &tm_v, n, cu);
    }
    if (warp == 0) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ prep (2 groups x 4 warps)
        // group g takes chunks n = g, g + 2, ...; warp wg of the group tokens 16wg .. 16wg+15;
        // lane: channels 8cg .. 8cg+7 (cg = lane % 8) of tokens tb .. tb+3 (tb = 16wg + 4rr,
        // rr = lane / 8).  Log-decay sums are in log2 units.
        const int g = warp / kGroupWarps, wg = warp % kGroupWarps;
        // lane 0 of the group's warps 0, 1, 2 issues, for chunk n of the group: the r / k / omega
        // copy of n+3, GU(n) and SC(n) (warp 0); GA(n-1) (warp 1); RO(n) (warp 2)
        const bool leader = wg == 0 && lane == 0;
        const bool ga_issuer = wg == 1 && lane == 0, ro_issuer = wg == 2 && lane == 0;
        const int cg = lane & 7, rr = lane >> 3;
        const int c0 = 8 * cg;
        const int tb = 16 * wg + 4 * rr;
        gw_check(status, tb + 3 < C && c0 + 8 <= 64);   // this thread's tokens / channels
        float2 uu[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            uu[q] = (kC2 || kQ) ? make_float2(0.f, 0.f) : make_float2(u[h * 64 + c0 + 2 * q], u[h * 64 + c0 + 2 * q + 1]);
        uint32_t toff[4];   // byte offset of this thread's 16-byte column in token row tb + p
#pragma unroll
        for (int p = 0; p < 4; ++p) toff[p] = (uint32_t)((tb + p) * 128 + ((cg ^ ((tb + p) & 7)) << 4));
        const float2 l2e = make_float2(kLog2e, kLog2e);
        const float2 nl2e = make_float2(-kLog2e, -kLog2e);
        bool issued = false;   // the leader issued tensor-core work (drained before exit)
        // GA(m) = Y[m & 1] += A(m) x V(m), issued by this group's leader for m = n - 1 (the other
        // group's chunk) once the epilogue stored A(m) and RO(m) (the other leader's) is complete
        auto issue_ga = [&](int m) {
            const int mb = m & 1;
            bool ok = wait_soft(s, &s.a_ready[mb], (uint32_t)((m >> 1) & 1), budget, m);
            ok = ok && wait_soft(s, &s.op_free[mb], (uint32_t)((m >> 1) & 1), budget, m);
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t ycol = tmem + COL_Y + 128 * mb;
                const uint32_t v_tile = ptx::smem_addr(s.vt[m % kStagesV]);
                const uint32_t at = ptx::smem_addr(s.at);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // Y += [A] x V
                    ptx::mma_bf16(ycol, ptx::desc_kmajor(at + 32 * kq),
                                  ptx::desc_mnmajor(v_tile + 2048 * kq), IDESC_GA, 1);
                issued = true;
                ptx::mma_commit(&s.ya_done[mb]);
            }
            // after a give-up (hand-over at or before m, or abort) nothing waits for chunk m's
            // phase, and completing it could alias an earlier phase a waiter has not seen
        };
        // RO(m) = Y[m & 1] = Rt(m) x S_{m-1}, for this group's chunk m, issued by warp 2 while
        // the group works on chunk m+2 (between its two passes), once the epilogue has stored
        // S_{m-1} in sb[m & 1] and read Y[m & 1] (end of its chunk m-1)
        int ro_next = g;   // this group's next chunk whose RO is to be issued
        auto issue_ro = [&](int m) {
            const int mb = m & 1;
            if (wait_soft(s, &s.s_ready[mb], (uint32_t)((m >> 1) & 1), budget, m)) {
                ptx::tc_fence_after();
                const uint32_t rtile = ptx::smem_addr(s.rt[mb]);
                const uint32_t sbuf = ptx::smem_addr(s.sb[mb]);
                const uint32_t ycol = tmem + COL_Y + 128 * mb;
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // Y = [Rt] x [S_hi^T ; S_lo^T]
                    ptx::mma_bf16(ycol, ptx::desc_kmajor(rtile + 32 * kq),
                                  ptx::desc_kmajor(sbuf + 32 * kq), IDESC_RO, kq > 0);
                issued = true;
                ptx::mma_commit(&s.op_free[mb]);
            }
            ro_next = m + kPrepGroups;
        };
        int n = g;
        for (; n < NC; n += kPrepGroups) {
            const int pb = n & 1, st = n % kStagesRkw;
            const int valid = min(C, T - (cseg + n) * C);
            // r / k / omega of chunk n; gamma / bonus slot n % 4, read by the epilogue for n-4
            bool ok_wait = wait_soft(s, &s.full_rkw[st], (uint32_t)((n / kStagesRkw) & 1), budget, n);
            if (n >= 4)
                ok_wait = ok_wait && wait_soft(s, &s.ep_free[n & 3], (uint32_t)(((n - 4) >> 2) & 1), budget, n);
            if (named_bar_any(kBarPrep0 + g, kGroupThreads, !ok_wait || stopped_at(s, n))) break;
            uint4 wv[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) wv[p] = lds128v(s.rkw[st][2], toff[p]);
            // pass 1: exp(omega) and the inclusive prefix of log2 w = -exp(omega) log2(e) over
            // this thread's 4 tokens
            float2 L[4][4];    // [token p][channel pair q]
            float2 acc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float2 e = exp2_2(__fmul2_rn(unpack2(word(wv[p], q)), l2e));
                    if (tb + p >= valid) e = make_float2(0.f, 0.f);
                    acc[q] = __ffma2_rn(e, nl2e, acc[q]);
                    L[p][q] = acc[q];
                }
            }
            // scan of the 4 run totals of the warp (lanes 8 apart), then the exclusive prefix
            float2 inc[4], exc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) inc[q] = acc[q];
#pragma unroll
            for (int d = 8; d <= 16; d <<= 1) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 o = shfl_up2(inc[q], d);
                    if (lane >= d) inc[q] = __fadd2_rn(inc[q], o);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 o = shfl_up2(inc[q], 8);
                exc[q] = rr > 0 ? o : make_float2(0.f, 0.f);
            }
            if (rr == 3) {   // warp totals for channels c0 .. c0+7
                float4* dst = reinterpret_cast<float4*>(&s.qtot[g][wg][cg][0]);
                dst[0] = make_float4(inc[0].x, inc[0].y, inc[1].x, inc[1].y);
                dst[1] = make_float4(inc[2].x, inc[2].y, inc[3].x, inc[3].y);
            }
            // Rt / Kh of parity pb were read by GU, SC and RO of chunk n-2, which this group
            // issued; RO(n-2) is issued now and committed on op_free[pb]
            if (ro_issuer && n >= kPrepGroups) issue_ro(n - kPrepGroups);
            __syncwarp();
            const bool ok_free = n < 2 || wait_soft(s, &s.op_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget, n);
            if (named_bar_any(kBarPrep0 + g, kGroupThreads, !ok_free)) break;
            float2 off[4], tot[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) off[q] = tot[q] = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kGroupWarps; ++w) {
                const float4* src = reinterpret_cast<const float4*>(&s.qtot[g][w][cg][0]);
                const float4 a0 = src[0], a1 = src[1];
                const float2 v[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w),
                                     make_float2(a1.x, a1.y), make_float2(a1.z, a1.w)};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (w < wg) off[q] = __fadd2_rn(off[q], v[q]);
                    tot[q] = __fadd2_rn(tot[q], v[q]);
                }
            }
            // every warp of the group sums the same totals in the same order, so all take
            // the same branch
            bool in_range = true;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                in_range = in_range && (tot[q].x >= -kMaxLog2Range) && (tot[q].y >= -kMaxLog2Range);
            if (!__all_sync(0xffffffffu, in_range)) {
                // hand this (b,h) to the level kernel from chunk n on (the other group may
                // have found a later chunk first: keep the earliest), and wake the epilogue.
                // The arrive completes the phase of mm_done[pb] for chunk n; it waits until
                // every epilogue thread is past its wait for chunk n-2 on the same barrier
                // (they have read DU of chunk n-1), or a parity wait there could see two
                // completed phases as none.  No arrive if the sequence stops earlier.
                if (leader) {
                    atomicMin(&s.stop_at, n);
                    const bool wake = n < 1 || wait_soft(s, &s.du_free, (uint32_t)((n - 1) & 1), budget, n - 1);
                    if (wake) mbar_arrive(&s.mm_done[pb]);
                }
                break;
            }
            if (wg == 0 && rr == 0) {
                float4* gdst = reinterpret_cast<float4*>(&s.gamma[n & 3][c0]);
                const float2 g0 = exp2_2(tot[0]), g1 = exp2_2(tot[1]), g2 = exp2_2(tot[2]),
                             g3 = exp2_2(tot[3]);
                gdst[0] = make_float4(g0.x, g0.y, g1.x, g1.y);
                gdst[1] = make_float4(g2.x, g2.y, g3.x, g3.y);
            }
            // absolute prefix: L of the token before the run, then L of each token
            float2 prev[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                prev[q] = __fadd2_rn(off[q], exc[q]);
#pragma unroll
                for (int p = 0; p < 4; ++p) L[p][q] = __fadd2_rn(prev[q], L[p][q]);
            }
            // pass 2: Rt = r 2^(L_{t-1}), Kh = k 2^(-L_t) as bf16 hi / lo; bonus partials
            uint8_t* rt = s.rt[pb];
            uint8_t* kh_hi = s.kh[pb];
            uint8_t* kh_lo = s.kh[pb] + kTile;
            float bon[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int t = tb + p;
                const uint32_t csw = (uint32_t)((cg ^ (t & 7)) << 4);
                const uint32_t hr = (uint32_t)hi_row(t) * 128 + csw;
                const uint4 rv = lds128v(s.rkw[st][0], toff[p]);
                const uint4 kv = lds128v(s.rkw[st][1], toff[p]);
                uint32_t rh[4], rl[4], khv[4], klv[4];
                float bsum = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 fr = exp2_2(prev[q]);
                    const float2 fk = exp2_2(make_float2(-L[p][q].x, -L[p][q].y));
                    prev[q] = L[p][q];
                    float2 rr2 = unpack2(word(rv, q));
                    float2 kk = unpack2(word(kv, q));
                    if (kC2 || kQ) {   // (1 - w), 1 - w = 1 - exp(-exp(omega)) without cancellation
                        float2 e = exp2_2(__fmul2_rn(unpack2(word(wv[p], q)), l2e));
                        if (t >= valid) e = make_float2(0.f, 0.f);
                        if (kC2) kk = __fmul2_rn(kk, one_minus_exp_neg2(e));   // key k (1 - w)
                        else rr2 = __fmul2_rn(rr2, one_minus_exp_neg2(e));     // query r (1 - w)
                    }
                    split2(__fmul2_rn(rr2, fr), rh[q], rl[q]);
                    split2(__fmul2_rn(kk, fk), khv[q], klv[q]);
                    if (!kC2) {
                        const float2 ru = __fmul2_rn(rr2, uu[q]);
                        bsum = fmaf(ru.x, kk.x, fmaf(ru.y, kk.y, bsum));
                    }
                }
                sts128(rt, hr, rh[0], rh[1], rh[2], rh[3]);
                sts128(rt, hr + 8 * 128, rl[0], rl[1], rl[2], rl[3]);
                sts128(kh_hi, toff[p], khv[0], khv[1], khv[2], khv[3]);
                sts128(kh_lo, toff[p], klv[0], klv[1], klv[2], klv[3]);
                bon[p] = bsum;
            }
            // bonus: reduce the 4 tokens' partials over the 8 channel columns (lane bits 0-2);
            // lane bit 2 then bit 1 pick the token each lane keeps
            if (!kC2) {
                const bool up2 = lane & 4, up1 = lane & 2;
                float k0 = (up2 ? bon[2] : bon[0]) + __shfl_xor_sync(0xffffffffu, up2 ? bon[0] : bon[2], 4);
                float k1 = (up2 ? bon[3] : bon[1]) + __shfl_xor_sync(0xffffffffu, up2 ? bon[1] : bon[3], 4);
                float kb = (up1 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, up1 ? k0 : k1, 2);
                kb += __shfl_xor_sync(0xffffffffu, kb, 1);
                if ((lane & 1) == 0) s.bonus[n & 3][tb + 2 * ((lane >> 2) & 1) + ((lane >> 1) & 1)] = kb;
            }
            ptx::fence_proxy_async_smem();
            // every thread of the group has read stage st and written its operands
            named_bar(kBarPrep0 + g, kGroupThreads);
            if (leader) {
                if (n + kStagesRkw < NC) load_rkw(s, &tm_r, &tm_k, &tm_w, n + kStagesRkw, cu);
                // GU(n), SC(n): v of chunk n; DU read by the epilogue for chunk n-1; the SC
                // buffer of parity pb read by A(n-2) (GA(n-2) waited for that).  Every wait
                // gives up if the sequence was handed over at or before the chunk it serves.
                bool ok = wait_soft(s, &s.full_v[n % kStagesV], (uint32_t)((n / kStagesV) & 1), budget, n);
                if (n >= 1) ok = ok && wait_soft(s, &s.du_free, (uint32_t)((n - 1) & 1), budget, n);
                if (ok) {
                    ptx::tc_fence_after();
                    const uint32_t v_tile = ptx::smem_addr(s.vt[n % kStagesV]);
                    const uint32_t kh = ptx::smem_addr(s.kh[pb]);
                    const uint32_t rtile = ptx::smem_addr(s.rt[pb]);
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)   // DU = V^T x [Kh_hi | Kh_lo]
                        ptx::mma_bf16(tmem + COL_DU, ptx::desc_mnmajor(v_tile + 2048 * kq),
                                      ptx::desc_sw128(kh + 2048 * kq, kTile), IDESC_GU, kq > 0);
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)   // SC = [Rt] x Kh_hi^T
                        ptx::mma_bf16(tmem + COL_SC + 64 * pb, ptx::desc_kmajor(rtile + 32 * kq),
                                      ptx::desc_kmajor(kh + 32 * kq), IDESC_SC, kq > 0);
                    ptx::mma_commit(&s.mm_done[pb]);
                    issued = true;
                }
            } else if (ga_issuer) {
                if (n >= 1) issue_ga(n - 1);
            }
            __syncwarp();
        }
        // the chunk this group stopped at (or the first past the sequence): GA of the chunk
        // before it is still this group's (it is the other group's chunk)
        if (ga_issuer && n >= 1 && n <= NC) issue_ga(n - 1);
        // RO of this group's last chunk whose products were issued
        if (ro_issuer && ro_next <= n - kPrepGroups && ro_next < NC) issue_ro(ro_next);
        // drain: this thread's tensor-core work must be complete before TMEM is freed
        if (issued) {   // one of the group's issuers
            ptx::mma_commit(&s.drain[g][wg]);
            ptx::mbar_wait(&s.drain[g][wg], 0, drain_budget);
        }
    } else {
        // ------------------------------------------------------------ epilogue (8 warps)
        // warp (q, ch0): TMEM sub-partition q = warp % 4, columns 32ch0 .. 32ch0+31 of each
        // 64-wide accumulator.  Thread: token / state rows r0 = 16q + l/4 and r1 = r0 + 8;
        // column pairs col0 + 8j + 2(l%4) + {0,1}, j = 0..3.
        const int q = warp & 3;
        const int ch0 = (warp - kEpiWarp0) >> 2;
        const int col0 = 32 * ch0, q0 = 4 * ch0;
        const int r0 = 16 * q + (lane >> 2), r1 = r0 + 8;
        const int cl = 2 * (lane & 3);
        gw_check(status, r1 < C && col0 + 8 * (kPairs - 1) + cl + 2 <= 64);   // rows, columns
        const uint32_t cb = (uint32_t)(lane & 3) * 4;
        const uint32_t lane_h0 = (uint32_t)(32 * q) << 16, lane_h1 = (uint32_t)(32 * q + 16) << 16;
        const int hr0 = hi_row(r0), hr1 = hi_row(r1);
        // A block of this warp: rows 16q..16q+15, columns 32ch0..32ch0+31
        const bool a_zero = 16 * q + 15 < col0;       // entirely above the diagonal
        const bool a_full = 16 * q >= col0 + 32;      // entirely below the diagonal
        const bool leader = tid == kEpiLeader;
        // state S[i][j] held transposed: rows j = r0, r1; columns i = col0 + 8j + cl + {0,1}
        float2 S0[kPairs], S1[kPairs];
        {
            const float* src = pseg > 0 ? seg.s_mid + ((size_t)bh * (seg.P - 1) + (pseg - 1)) * 4096
                                     : s_in ? s_in + (size_t)bh * 4096 : nullptr;
#pragma unroll
            for (int j = 0; j < kPairs; ++j) {
                const int i = col0 + 8 * j + cl;
                S0[j] = src ? make_float2(src[i * 64 + r0], src[(i + 1) * 64 + r0]) : make_float2(0.f, 0.f);
                S1[j] = src ? make_float2(src[i * 64 + r1], src[(i + 1) * 64 + r1]) : make_float2(0.f, 0.f);
            }
            store_state(s.sb[0], S0, S1, r0, r1, q0, cb);   // S entering chunk 0, read by RO(0)
            if (a_zero) {                     // blocks of A that are always zero: once, here
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sts32(s.at, sw_off(hr0, q0 + k) + cb, 0u);
                    sts32(s.at, sw_off(hr0 + 8, q0 + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1, q0 + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1 + 8, q0 + k) + cb, 0u);
                }
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.s_ready[0]);   // RO(0) may run
        }
        if (kGN && tid - kEpiLeader < 64) {   // read by output_chunk after the epilogue's barriers
            s.gn_gamma[tid - kEpiLeader] = gn.gamma[h * 64 + tid - kEpiLeader];
            s.gn_beta[tid - kEpiLeader] = gn.beta[h * 64 + tid - kEpiLeader];
        }
        uint32_t up0[kPairs], up1[kPairs];   // Finch-C2: u' (GroupNorm: the gate) of the next output
#pragma unroll
        for (int j = 0; j < kPairs; ++j) up0[j] = up1[j] = 0u;
        int n = 0;
        for (; n < NC; ++n) {
            const int pb = n & 1;
            // Finch-C2: u' of chunk n-1 is read from HBM now and used by output(n-1) below
            // (GroupNorm: the gate of chunk n-1, the same way)
            if ((kC2 || kGN) && n >= 1)
                load_uprime(kGN ? static_cast<const __nv_bfloat16*>(gn.gate) : uprime, n - 1, cseg, b,
                            h, T, H, col0, cl, r0, r1, up0, up1);
            // ---- state(n): S <- gamma (S + DU), DU^T[j][i] accumulated on the tensor cores.
            // gamma and bonus of chunk n reach us through prep's named barrier -> its leader's
            // MMA issue -> the commit on mm_done (or, at a hand-over, the leader's arrive).
            {
                const bool ok = wait_soft(s, &s.mm_done[pb], (uint32_t)((n >> 1) & 1), budget);
                // uniform over the epilogue: stop (hand-off) or abort
                if (named_bar_any(kBarEpi, kEpiThreads, !ok || stopped_at(s, n))) break;
            }
            ptx::tc_fence_after();
            {
                uint32_t ua[16], ub[16];
                tmem_ld16x4(tmem + lane_h0 + COL_DU + col0, ua);
                tmem_ld16x4(tmem + lane_h0 + COL_DU + 64 + col0, ub);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                mbar_arrive(&s.du_free);
                const float* gam = s.gamma[n & 3] + col0 + cl;
#pragma unroll
                for (int j = 0; j < kPairs; ++j) {
                    const float2 gg = *reinterpret_cast<const float2*>(gam + 8 * j);
                    S0[j] = __fmul2_rn(gg, __fadd2_rn(S0[j], __fadd2_rn(lo_pair(ua, j), lo_pair(ub, j))));
                    S1[j] = __fmul2_rn(gg, __fadd2_rn(S1[j], __fadd2_rn(hi_pair(ua, j), hi_pair(ub, j))));
                }
            }
            // RO(n-1) read sb[(n+1) & 1] and GA(n-1) the A tile: both are done once the commit
            // after GA(n-1) has landed (which also lets output(n-1) read Y below)
            if (n >= 1 && !wait_soft(s, &s.ya_done[(n - 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), budget))
                s.abort = 1;
            if (n + 1 < NC) store_state(s.sb[(n + 1) & 1], S0, S1, r0, r1, q0, cb);   // for RO(n+1)
            // ---- A(n): masked scores with the bonus on the diagonal, hi / lo, for GA(n).  SC(n)
            // is complete: it was committed with GU(n) on mm_done.
            if (!a_zero) {
                uint32_t p0[16], p1[16];
                tmem_ld16x4(tmem + lane_h0 + COL_SC + 64 * pb + col0, p0);
                tmem_ld16x4(tmem + lane_h1 + COL_SC + 64 * pb + col0, p1);
                ptx::tmem_wait_ld();
                const float b0 = kC2 ? 0.f : s.bonus[n & 3][r0], b1 = kC2 ? 0.f : s.bonus[n & 3][r1];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 a0 = rows_sum(p0, k), a1 = rows_sum(p1, k);
                    if (!a_full) {   // strictly causal scores, bonus on the diagonal
                        const int sx = col0 + 8 * k + cl;
                        a0.x = sx < r0 ? a0.x : (sx == r0 ? b0 : 0.f);
                        a0.y = sx + 1 < r0 ? a0.y : (sx + 1 == r0 ? b0 : 0.f);
                        a1.x = sx < r1 ? a1.x : (sx == r1 ? b1 : 0.f);
                        a1.y = sx + 1 < r1 ? a1.y : (sx + 1 == r1 ? b1 : 0.f);
                    }
                    uint32_t hi, lo;
                    split2(a0, hi, lo);
                    sts32(s.at, sw_off(hr0, q0 + k) + cb, hi);
                    sts32(s.at, sw_off(hr0 + 8, q0 + k) + cb, lo);
                    split2(a1, hi, lo);
                    sts32(s.at, sw_off(hr1, q0 + k) + cb, hi);
                    sts32(s.at, sw_off(hr1 + 8, q0 + k) + cb, lo);
                }
            }
            // A(n) (and S_n) stored, SC(n), gamma and bonus of chunk n read: GA(n) may run
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            mbar_arrive(&s.ep_free[n & 3]);
            mbar_arrive(&s.a_ready[pb]);
            // ---- output of chunk n-1 (GA(n-1) is complete: waited above)
            if (n >= 1) {
                ptx::tc_fence_after();
                output_chunk<kC2, kGN>(s, gn.eps, n - 1, cseg, tmem, lane_h0, lane_h1, col0, cl, r0, r1, b, h, T, H, y,
                                  y_raw, up0, up1);
                // v stage (n+3) % 4 held v(n-1), read by GU(n-1) and GA(n-1), both complete
                if (leader && n + kStagesV - 1 < NC && !stopped_at(s, n + kStagesV - 1))
                    load_v(s, &tm_v, n + kStagesV - 1, cu);
            }
            // S_n is in sb[(n+1) & 1] and Y[(n+1) & 1] (output(n-1)) has been read: RO(n+1)
            ptx::tc_fence_before();
            mbar_arrive(&s.s_ready[(n + 1) & 1]);
        }
        // ---- leave: output of the last chunk done, final state (or the state entering the
        // chunk handed to the level kernel)
        if (n >= 1) {
            const bool ok = wait_soft(s, &s.ya_done[(n - 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), budget);
            // uniform over the epilogue (the GroupNorm stage synchronises warp pairs)
            if (!named_bar_any(kBarEpi, kEpiThreads, !ok || ld_volatile(&s.abort) != 0)) {
                if (kC2 || kGN)
                    load_uprime(kGN ? static_cast<const __nv_bfloat16*>(gn.gate) : uprime, n - 1, cseg,
                                b, h, T, H, col0, cl, r0, r1, up0, up1);
                ptx::tc_fence_after();
                output_chunk<kC2, kGN>(s, gn.eps, n - 1, cseg, tmem, lane_h0, lane_h1, col0, cl, r0, r1, b, h, T, H, y,
                                  y_raw, up0, up1);
            }
        }
        const bool aborted = ld_volatile(&s.abort) != 0;
        if (!aborted) {
            const bool stopped = (n < NC);
            float* dst = stopped                       ? handoff_state + (size_t)unit * 4096
                         : (s_out && pseg == seg.P - 1) ? s_out + (size_t)bh * 4096
                                                     : nullptr;
            if (dst) {
#pragma unroll
                for (int j = 0; j < kPairs; ++j) {
                    const int i = col0 + 8 * j + cl;
                    dst[i * 64 + r0] = S0[j].x;
                    dst[(i + 1) * 64 + r0] = S0[j].y;
                    dst[i * 64 + r1] = S1[j].x;
                    dst[(i + 1) * 64 + r1] = S1[j].y;
                }
            }
            if (leader) handoff_chunk[unit] = stopped ? cseg + n : -1;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // every issued copy must land before the CTA may exit
        for (int st = 0; st < kStagesRkw; ++st)
            if (s.last_rkw[st] >= 0)
                ptx::mbar_wait(&s.full_rkw[st], (uint32_t)((s.last_rkw[st] / kStagesRkw) & 1), drain_budget);
        for (int st = 0; st < kStagesV; ++st)
            if (s.last_v[st] >= 0)
                ptx::mbar_wait(&s.full_v[st], (uint32_t)((s.last_v[st] / kStagesV) & 1), drain_budget);
        if (s.abort) {
            atomicExch(status, 1);
            handoff_chunk[unit] = -1;
        }
    }
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

size_t fast_smem_bytes() { return sizeof(Smem) + 1024; }
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "the fast kernel's shared memory exceeds a CTA's 227 KB");

cudaError_t launch_chunked_fast(const CUtensorMap* maps, const float* u, const float* s_in,
                                float* s_out, void* y, float* y_raw, int B, int T, int H,
                                Segments seg, Variant var, int* status, int* handoff_chunk,
                                float* handoff_state, long long budget, cudaStream_t st,
                                const GnOut* gn) {
    const size_t smem = fast_smem_bytes();
    auto kernel = var.uprime     ? wkv6_fast_kernel<true, false, false>
                  : gn           ? wkv6_fast_kernel<false, true, false>
                  : var.query_c2 ? wkv6_fast_kernel<false, false, true>
                                 : wkv6_fast_kernel<false, false, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const GnOut g = gn ? *gn : GnOut{nullptr, nullptr, 0.f, nullptr};
    kernel<<<(unsigned)(B * H * seg.P), kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], u, s_in, s_out, static_cast<__nv_bfloat16*>(y),
        y_raw, static_cast<const __nv_bfloat16*>(var.uprime), g, T, H, seg, status, handoff_chunk,
        handoff_state, budget, 4000000000LL);
    return cudaGetLastError();
}

}  // namespace goldwkv
