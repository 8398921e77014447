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
// split for the state increment.  The lo parts cost no extra MMA instructions: hi and lo
// rows are stacked into M = 128 (rows 0-7 of every 16-row group hold hi parts of 8 tokens,
// rows 8-15 the lo parts of the same tokens), and a 16x256b TMEM load hands each thread the
// hi and lo element of the same (token, column) in registers {0,1} / {2,3}, so the
// combination is one add in registers.
//
// The recurrence and the output are separate pipelines.  The state only needs
//   GU(n): V^T (M=64) x [Kh_hi | Kh_lo] (N=128) -> DU = (Kh^T V)^T, the increment of chunk n,
// which depends on the chunk's own operands, not on S; the epilogue folds it into the fp32
// state it keeps in registers.  The output of chunk n needs three more products:
//   SC(n): [Rt_hi ; Rt_lo] (M=128) x Kh_hi^T (N=64)           intra-chunk scores
//   RO(n): [Rt_hi ; Rt_lo] x [S_hi^T ; S_lo^T] (N=128)        readout of S_{n-1} -> Y
//   GA(n): [A_hi ; A_lo] x V (N=64), accumulated into Y        A = masked scores + bonus
// None of them feeds back into S, so they trail the state by a chunk without stalling it.
//
// Warp roles (608 threads):
//   warp 0, one thread: TMA loads (3-stage rings: r/k/omega released by prep, v by GU and GA);
//     TMEM owner.
//   warp 1, one thread: GU(n), SC(n) in chunk order.  warp 2, one thread: RO(n), GA(n).  Each
//     blocks on the one barrier it needs next; two issuers let the state stream run ahead
//     of the output stream.  Buffers read by both are released by one commit from each.
//   warps 3-10 (prep): 8 tokens each of the same chunk -- log-decay prefix, Rt / Kh hi/lo
//     operands, bonus, gamma, range test.
//   warps 11-18 (epilogue): per chunk n, state(n) = gamma (S + DU) and S_n hi/lo for RO(n+1);
//     the output of chunk n-1 (Y -> y); A(n) for GA(n).
// Handshakes are mbarriers; every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "chunk_tiles.cuh"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

using namespace tiles;

constexpr int C = 64;
constexpr int kStages = 3;
constexpr int kPrepWarps = 8, kEpiWarps = 8;
constexpr int kTok = C / kPrepWarps;   // tokens per prep warp (a power of two <= 32)
constexpr int kTmaWarp = 0, kMmaUWarp = 1, kMmaYWarp = 2;
constexpr int kPrepWarp0 = 3, kEpiWarp0 = kPrepWarp0 + kPrepWarps;
constexpr int kPrepThreads = 32 * kPrepWarps, kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 32 * kPrepWarp0 + kPrepThreads + kEpiThreads;
constexpr uint32_t kTmemCols = 512;
// DU: 2 buffers x 128 columns (M=64); SC: 2 x 64 (M=128); Y: 128 (M=128)
constexpr uint32_t COL_DU = 0, COL_SC = 256, COL_Y = 384;
// log2 of the largest factor exp(-L_s) allowed: ln range 60 -> log2 range 86.56
constexpr float kMaxLog2Range = 86.5617f;
constexpr float kLog2e = 1.4426950408889634f;
// named barriers (id 0 is __syncthreads)
constexpr int kBarPrep = 1, kBarEpi = 2;

constexpr uint32_t IDESC_GU = ptx::idesc_bf16(64, 128, 1, 1);
constexpr uint32_t IDESC_SC = ptx::idesc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_RO = ptx::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t IDESC_GA = ptx::idesc_bf16(128, 64, 0, 1);

struct __align__(1024) Smem {
    uint8_t rkw[kStages][3][kTile];  // r, k, omega tiles (TMA, 128B swizzle)
    uint8_t vt[kStages][kTile];      // v tiles
    uint8_t rt[2][2 * kTile];        // per parity: Rt hi/lo, 128 stacked rows
    uint8_t kh[2][2 * kTile];        // per parity: Kh_hi tile, then Kh_lo tile
    uint8_t sb[2][2 * kTile];        // S_hi^T tile, then S_lo^T tile; sb[m & 1] feeds RO(m)
    uint8_t at[2 * kTile];           // A hi/lo, 128 stacked rows
    float qtot[2][kPrepWarps][64];   // prep: per-warp sums of log2 w
    float gamma[2][64];
    float bonus[2][64];
    int unsafe[2];
    uint64_t full_rkw[kStages], empty_rkw[kStages], full_v[kStages], empty_v[kStages];
    uint64_t prep_done[2], op_free[2], ep_free[2];
    uint64_t gu_done[2], sc_done[2], du_free[2], sc_free[2], s_ready[2], s_free[2];
    uint64_t a_ready, ya_done, y_free;
    uint32_t tmem_base;
    int abort;
    int stop_at;                     // chunk at which this (b,h) leaves for the level kernel
};

// Output of chunk m (plus the second value u' of Finch-C2, whose words up0 / up1 for rows
// r0 / r1 the caller loaded ahead of time): y = Y[:, 0:64] + Y[:, 64:128] (hi and lo rows each), stored as bf16 (or
// fp32 rows to y_raw).  Frees the Y accumulator for RO(m+1).
template <bool kC2>
__device__ __forceinline__ void output_chunk(Smem& s, int m, int c0, uint32_t tmem, uint32_t lane_h0,
                                             uint32_t lane_h1, int ch, int cbase, int r0, int r1,
                                             int b, int h, int T, int H, __nv_bfloat16* y,
                                             float* y_raw, const uint32_t (&up0)[4],
                                             const uint32_t (&up1)[4], long long budget) {
    // m: chunk index within the unit (GA(m) is the (m+1)-th ya_done phase); c0 + m: absolute
    wait_soft(s, &s.ya_done, (uint32_t)(m & 1), budget);
    ptx::tc_fence_after();
    float2 Y0[4], Y1[4];
    {
        uint32_t a[16], c[16];
        tmem_ld16x4(tmem + lane_h0 + COL_Y + 32 * ch, a);
        tmem_ld16x4(tmem + lane_h0 + COL_Y + 64 + 32 * ch, c);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) Y0[k] = __fadd2_rn(rows_sum(a, k), rows_sum(c, k));
    }
    {
        uint32_t a[16], c[16];
        tmem_ld16x4(tmem + lane_h1 + COL_Y + 32 * ch, a);
        tmem_ld16x4(tmem + lane_h1 + COL_Y + 64 + 32 * ch, c);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) Y1[k] = __fadd2_rn(rows_sum(a, k), rows_sum(c, k));
    }
    ptx::tc_fence_before();
    mbar_arrive(&s.y_free);
    const int tc = (c0 + m) * C;
    const int valid = min(C, T - tc);
    const size_t row0 = ((size_t)b * T + (size_t)tc + r0) * H + h;
    const size_t row1 = ((size_t)b * T + (size_t)tc + r1) * H + h;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int j = cbase + 8 * k;
        if (kC2) {   // Finch-C2: the second value u'_t joins the readout (loaded beforehand)
            Y0[k] = __fadd2_rn(Y0[k], unpack2(up0[k]));
            Y1[k] = __fadd2_rn(Y1[k], unpack2(up1[k]));
        }
        if (y_raw != nullptr) {
            if (r0 < valid) *reinterpret_cast<float2*>(y_raw + row0 * 64 + j) = Y0[k];
            if (r1 < valid) *reinterpret_cast<float2*>(y_raw + row1 * 64 + j) = Y1[k];
        } else {
            if (r0 < valid) *reinterpret_cast<uint32_t*>(y + row0 * 64 + j) = pack2(Y0[k].x, Y0[k].y);
            if (r1 < valid) *reinterpret_cast<uint32_t*>(y + row1 * 64 + j) = pack2(Y1[k].x, Y1[k].y);
        }
    }
}

// u' words of chunk (c0 + m) for this thread's rows r0, r1 and column pairs cbase + 8k;
// rows past T read as zero.  Issued well before output_chunk needs them.
__device__ __forceinline__ void load_uprime(const __nv_bfloat16* __restrict__ uprime, int m, int c0,
                                            int b, int h, int T, int H, int cbase, int r0, int r1,
                                            uint32_t (&up0)[4], uint32_t (&up1)[4]) {
    const int tc = (c0 + m) * C;
    const int valid = min(C, T - tc);
    const size_t row0 = ((size_t)b * T + (size_t)tc + r0) * H + h;
    const size_t row1 = ((size_t)b * T + (size_t)tc + r1) * H + h;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int j = cbase + 8 * k;
        up0[k] = r0 < valid ? __ldg(reinterpret_cast<const unsigned int*>(uprime + row0 * 64 + j)) : 0u;
        up1[k] = r1 < valid ? __ldg(reinterpret_cast<const unsigned int*>(uprime + row1 * 64 + j)) : 0u;
    }
}

// S_hi^T at tile, S_lo^T at tile + kTile: this thread's rows j = r0, r1, columns i of its pairs
__device__ __forceinline__ void store_state(uint8_t* tile, const float2 (&S0)[4], const float2 (&S1)[4],
                                            int r0, int r1, int ch, uint32_t cb) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t hi, lo;
        split2(S0[k], hi, lo);
        sts32(tile, sw_off(r0, 4 * ch + k) + cb, hi);
        sts32(tile + kTile, sw_off(r0, 4 * ch + k) + cb, lo);
        split2(S1[k], hi, lo);
        sts32(tile, sw_off(r1, 4 * ch + k) + cb, hi);
        sts32(tile + kTile, sw_off(r1, 4 * ch + k) + cb, lo);
    }
}

// kC2: Finch-C2 exact form -- key k (1 - w), no static bonus, second value uprime added.
template <bool kC2>
__global__ void __launch_bounds__(kThreads, 1)
wkv6_fast_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                 const float* __restrict__ u, const float* s_in, float* s_out,
                 __nv_bfloat16* __restrict__ y, float* __restrict__ y_raw,
                 const __nv_bfloat16* __restrict__ uprime, int T, int H,
                 Segments seg, int* status, int* handoff_chunk, float* handoff_state,
                 long long budget, long long drain_budget) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // unit: segment pseg of sequence bh; chunks cseg .. cseg + NC - 1 (absolute indices)
    const int unit = blockIdx.x, nbh = gridDim.x / seg.P;
    const int bh = unit % nbh, pseg = unit / nbh, b = bh / H, h = bh - (bh / H) * H;
    const int cseg = pseg * seg.seg_chunks;
    const int NC = min((T + C - 1) / C, cseg + seg.seg_chunks) - cseg;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&s.full_rkw[i], 1);
            ptx::mbar_init(&s.empty_rkw[i], kPrepThreads);
            ptx::mbar_init(&s.full_v[i], 1);
            ptx::mbar_init(&s.empty_v[i], 2);      // GU (warp 1) and GA (warp 2)
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.prep_done[i], kPrepThreads);
            ptx::mbar_init(&s.op_free[i], 2);      // GU/SC (warp 1) and RO (warp 2)
            ptx::mbar_init(&s.ep_free[i], kEpiThreads);
            ptx::mbar_init(&s.gu_done[i], 1);
            ptx::mbar_init(&s.sc_done[i], 1);
            ptx::mbar_init(&s.du_free[i], kEpiThreads);
            ptx::mbar_init(&s.sc_free[i], kEpiThreads);
            ptx::mbar_init(&s.s_ready[i], kEpiThreads);
            ptx::mbar_init(&s.s_free[i], 1);
        }
        ptx::mbar_init(&s.a_ready, kEpiThreads);
        ptx::mbar_init(&s.ya_done, 1);
        ptx::mbar_init(&s.y_free, kEpiThreads);
        ptx::fence_mbar_init();
        s.abort = 0;
        s.stop_at = -1;
    }
    if (warp == kTmaWarp) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_r);
            ptx::prefetch_tensormap(&tm_k);
            ptx::prefetch_tensormap(&tm_v);
            ptx::prefetch_tensormap(&tm_w);
            int last_rkw[kStages] = {-1, -1, -1}, last_v[kStages] = {-1, -1, -1};
            for (int n = 0; n < NC; ++n) {
                const int st = n % kStages;
                const uint32_t par = (uint32_t)((n / kStages - 1) & 1);   // release of chunk n-3
                if (n >= kStages && !wait_soft(s, &s.empty_rkw[st], par, budget, true)) break;
                ptx::mbar_arrive_expect_tx(&s.full_rkw[st], 3 * kTile);
                ptx::tma_load_4d(s.rkw[st][0], &tm_r, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
                ptx::tma_load_4d(s.rkw[st][1], &tm_k, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
                ptx::tma_load_4d(s.rkw[st][2], &tm_w, &s.full_rkw[st], 0, h, (cseg + n) * C, b);
                last_rkw[st] = n;
                if (n >= kStages && !wait_soft(s, &s.empty_v[st], par, budget, true)) break;
                ptx::mbar_arrive_expect_tx(&s.full_v[st], kTile);
                ptx::tma_load_4d(s.vt[st], &tm_v, &s.full_v[st], 0, h, (cseg + n) * C, b);
                last_v[st] = n;
            }
            // every issued copy must land before the CTA may exit
            for (int st = 0; st < kStages; ++st) {
                if (last_rkw[st] >= 0)
                    ptx::mbar_wait(&s.full_rkw[st], (uint32_t)((last_rkw[st] / kStages) & 1), drain_budget);
                if (last_v[st] >= 0)
                    ptx::mbar_wait(&s.full_v[st], (uint32_t)((last_v[st] / kStages) & 1), drain_budget);
            }
        }
    } else if (warp == kMmaUWarp) {
        // ------------------------------------------------------------ GU, SC issue
        if (lane == 0) {
            int last = -1;
            for (int n = 0; n < NC; ++n) {
                const int pb = n & 1, st = n % kStages;
                if (!wait_soft(s, &s.prep_done[pb], (uint32_t)((n >> 1) & 1), budget)) break;
                if (ld_volatile(&s.unsafe[pb])) {   // hand this (b,h) to the level kernel
                    s.stop_at = n;
                    mbar_arrive(&s.gu_done[pb]);    // wakes the epilogue, which hands off
                    break;
                }
                if (!wait_soft(s, &s.full_v[st], (uint32_t)((n / kStages) & 1), budget)) break;
                if (n >= 2 && !wait_soft(s, &s.du_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget)) break;
                if (n >= 2 && !wait_soft(s, &s.sc_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget)) break;
                ptx::tc_fence_after();
                const uint32_t v_tile = ptx::smem_addr(s.vt[st]);
                const uint32_t kh = ptx::smem_addr(s.kh[pb]);
                const uint32_t rt = ptx::smem_addr(s.rt[pb]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // DU = V^T x [Kh_hi | Kh_lo]
                    ptx::mma_bf16(tmem + COL_DU + 128 * pb, ptx::desc_sw128(v_tile + 2048 * kq, 1024),
                                  ptx::desc_sw128(kh + 2048 * kq, kTile), IDESC_GU, kq > 0);
                ptx::mma_commit(&s.gu_done[pb]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // SC = [Rt] x Kh_hi^T
                    ptx::mma_bf16(tmem + COL_SC + 64 * pb, ptx::desc_kmajor(rt + 32 * kq),
                                  ptx::desc_kmajor(kh + 32 * kq), IDESC_SC, kq > 0);
                ptx::mma_commit(&s.sc_done[pb]);
                ptx::mma_commit(&s.op_free[pb]);
                ptx::mma_commit(&s.empty_v[st]);
                last = n;
            }
            // drain: our tensor-core work must be complete before TMEM is freed
            if (last >= 0) ptx::mbar_wait(&s.sc_done[last & 1], (uint32_t)((last >> 1) & 1), drain_budget);
        }
    } else if (warp == kMmaYWarp) {
        // ------------------------------------------------------------ RO, GA issue
        if (lane == 0) {
            uint64_t* last_bar = nullptr;   // the latest commit covers all earlier MMAs
            uint32_t last_par = 0;
            for (int n = 0; n < NC; ++n) {
                const int pb = n & 1, st = n % kStages;
                if (!wait_soft(s, &s.prep_done[pb], (uint32_t)((n >> 1) & 1), budget)) break;
                if (ld_volatile(&s.unsafe[pb])) break;   // chunks before n are complete
                if (!wait_soft(s, &s.s_ready[pb], (uint32_t)((n >> 1) & 1), budget)) break;
                if (n >= 1 && !wait_soft(s, &s.y_free, (uint32_t)((n - 1) & 1), budget)) break;
                ptx::tc_fence_after();
                const uint32_t rt = ptx::smem_addr(s.rt[pb]);
                const uint32_t sbuf = ptx::smem_addr(s.sb[pb]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // Y = [Rt] x [S_hi^T ; S_lo^T]
                    ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(rt + 32 * kq),
                                  ptx::desc_kmajor(sbuf + 32 * kq), IDESC_RO, kq > 0);
                ptx::mma_commit(&s.s_free[pb]);    // sb[pb] read
                ptx::mma_commit(&s.op_free[pb]);   // Rt of parity pb read
                last_bar = &s.s_free[pb];
                last_par = (uint32_t)((n >> 1) & 1);
                if (!wait_soft(s, &s.a_ready, (uint32_t)(n & 1), budget)) break;
                ptx::tc_fence_after();
                const uint32_t v_tile = ptx::smem_addr(s.vt[st]);
                const uint32_t at = ptx::smem_addr(s.at);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // Y[:, 0:64] += [A] x V
                    ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(at + 32 * kq),
                                  ptx::desc_mnmajor(v_tile + 2048 * kq), IDESC_GA, 1);
                ptx::mma_commit(&s.ya_done);
                ptx::mma_commit(&s.empty_v[st]);
                last_bar = &s.ya_done;
                last_par = (uint32_t)(n & 1);
            }
            if (last_bar != nullptr) ptx::mbar_wait(last_bar, last_par, drain_budget);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ prep (8 warps)
        // warp g: tokens 8g .. 8g+7 of every chunk; lane = channel pair (2l, 2l+1); log2 units
        const int g = warp - kPrepWarp0;
        const int c0 = 2 * lane;
        const float2 uu = kC2 ? make_float2(0.f, 0.f) : make_float2(u[h * 64 + c0], u[h * 64 + c0 + 1]);
        const int chunk = lane >> 2;          // 16-byte chunk holding channels c0, c0+1
        const uint32_t cbyte = (uint32_t)(lane & 3) * 4;
        const float2 l2e = make_float2(kLog2e, kLog2e);
        const float2 nl2e = make_float2(-kLog2e, -kLog2e);
        for (int n = 0; n < NC; ++n) {
            const int pb = n & 1, st = n % kStages;
            const int valid = min(C, T - (cseg + n) * C);
            bool ok_wait = wait_soft(s, &s.full_rkw[st], (uint32_t)((n / kStages) & 1), budget);
            if (n >= 2) {
                ok_wait = ok_wait && wait_soft(s, &s.op_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget);
                ok_wait = ok_wait && wait_soft(s, &s.ep_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget);
            }
            if (named_bar_any(kBarPrep, kPrepThreads, !ok_wait || ld_volatile(&s.abort))) break;
            const uint8_t* r_tile = s.rkw[st][0];
            const uint8_t* k_tile = s.rkw[st][1];
            const uint8_t* w_tile = s.rkw[st][2];
            // pass 1: local inclusive prefix of log2 w = -exp(omega) log2(e)
            float2 L[kTok];
            float2 ex[kTok];   // exp(omega) of each token (Finch-C2 normalises the key with it)
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int p = 0; p < kTok; ++p) {
                const int t = kTok * g + p;
                const float2 om = __fmul2_rn(unpack2(lds32(w_tile, sw_off(t, chunk) + cbyte)), l2e);
                float2 e = make_float2(fast_exp2(om.x), fast_exp2(om.y));
                if (t >= valid) e = make_float2(0.f, 0.f);
                acc = __ffma2_rn(e, nl2e, acc);
                L[p] = acc;
                ex[p] = e;
            }
            *reinterpret_cast<float2*>(&s.qtot[pb][g][c0]) = acc;
            named_bar(kBarPrep, kPrepThreads);
            float2 off = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kPrepWarps; ++w) {
                const float2 qv = *reinterpret_cast<const float2*>(&s.qtot[pb][w][c0]);
                if (w < g) off = __fadd2_rn(off, qv);
                tot = __fadd2_rn(tot, qv);
            }
            // every warp sees the same totals, so all take the same branch
            const bool ok = __all_sync(0xffffffffu, (tot.x >= -kMaxLog2Range) && (tot.y >= -kMaxLog2Range));
            if (!ok) {
                if (g == 0 && lane == 0) s.unsafe[pb] = 1;
                mbar_arrive(&s.prep_done[pb]);
                break;                        // this (b,h) continues in the level kernel
            }
            // pass 2: Rt = r 2^(L_{t-1}), Kh = k 2^(-L_t) as bf16 hi / lo; bonus partials
            uint32_t rw[kTok], kw[kTok];
#pragma unroll
            for (int p = 0; p < kTok; ++p) {
                const uint32_t o = sw_off(kTok * g + p, chunk) + cbyte;
                rw[p] = lds32(r_tile, o);
                kw[p] = lds32(k_tile, o);
            }
            mbar_arrive(&s.empty_rkw[st]);   // r, k, omega of this stage read
            uint8_t* rt = s.rt[pb];
            uint8_t* kh_hi = s.kh[pb];
            uint8_t* kh_lo = s.kh[pb] + kTile;
            // all exponentials first (independent of each other), then products and stores
            float2 fr[kTok], fk[kTok];   // 2^(L_{t-1}), 2^(-L_t)
            fr[0] = make_float2(fast_exp2(off.x), fast_exp2(off.y));
#pragma unroll
            for (int p = 0; p < kTok; ++p) {
                const float2 li = __fadd2_rn(off, L[p]);
                fk[p] = make_float2(fast_exp2(-li.x), fast_exp2(-li.y));
                if (p < kTok - 1) fr[p + 1] = make_float2(fast_exp2(li.x), fast_exp2(li.y));
            }
            float bon[kTok];
#pragma unroll
            for (int p = 0; p < kTok; ++p) {
                const int t = kTok * g + p;
                const uint32_t o = sw_off(t, chunk) + cbyte;
                const float2 rr = unpack2(rw[p]);
                float2 kk = unpack2(kw[p]);
                if (kC2)   // k (1 - w), 1 - w = 1 - exp(-exp(omega)) without cancellation
                    kk = __fmul2_rn(kk, one_minus_exp_neg2(ex[p]));
                uint32_t hi, lo;
                split2(__fmul2_rn(rr, fr[p]), hi, lo);
                const int hr = hi_row(t);
                const uint32_t cb = (uint32_t)(chunk ^ (t & 7)) << 4;
                sts32(rt, (uint32_t)hr * 128 + cb + cbyte, hi);
                sts32(rt, (uint32_t)(hr + 8) * 128 + cb + cbyte, lo);
                split2(__fmul2_rn(kk, fk[p]), hi, lo);
                sts32(kh_hi, o, hi);
                sts32(kh_lo, o, lo);
                if (!kC2) {
                    const float2 ru = __fmul2_rn(rr, uu);
                    bon[p] = fmaf(ru.x, kk.x, ru.y * kk.y);
                }
            }
            // bonus: reduce the kTok per-token partials over the 32 lanes (reduce-scatter: each
            // halving step keeps half of the tokens on each side of a lane-bit split)
            if (!kC2) {
                constexpr int kSteps = kTok == 8 ? 3 : kTok == 4 ? 2 : kTok == 2 ? 1 : 0;
#pragma unroll
                for (int stp = 0; stp < kSteps; ++stp) {
                    const int mask = 16 >> stp, half = kTok >> (stp + 1);
                    const bool up = lane & mask;
#pragma unroll
                    for (int i = 0; i < half; ++i) {
                        const float send = up ? bon[i] : bon[i + half];
                        const float keep = up ? bon[i + half] : bon[i];
                        bon[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                    }
                }
#pragma unroll
                for (int mask = 16 >> kSteps; mask >= 1; mask >>= 1)
                    bon[0] += __shfl_xor_sync(0xffffffffu, bon[0], mask);
                if ((lane & ((32 >> kSteps) - 1)) == 0) {
                    int p = 0;   // token index: lane bits 4, 3, ... of the halving steps
#pragma unroll
                    for (int stp = 0; stp < kSteps; ++stp) p = 2 * p + ((lane >> (4 - stp)) & 1);
                    s.bonus[pb][kTok * g + p] = bon[0];
                }
            }
            if (g == 0) {
                *reinterpret_cast<float2*>(&s.gamma[pb][c0]) = make_float2(fast_exp2(tot.x), fast_exp2(tot.y));
                if (lane == 0) s.unsafe[pb] = 0;
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.prep_done[pb]);
        }
    } else {
        // ------------------------------------------------------------ epilogue (8 warps)
        // warp (q, ch): TMEM sub-partition q = warp % 4, columns 32ch .. 32ch+31 of each
        // 64-wide block.  Thread: token / state rows r0 = 16q + l/4 and r1 = r0 + 8; column
        // pairs cbase + 8k + {0,1}, k = 0..3.
        const int q = warp & 3;
        const int ch = (warp - kEpiWarp0) >> 2;
        const int r0 = 16 * q + (lane >> 2), r1 = r0 + 8;
        const int cbase = 32 * ch + 2 * (lane & 3);
        const uint32_t cb = (uint32_t)(lane & 3) * 4;
        const uint32_t lane_h0 = (uint32_t)(32 * q) << 16, lane_h1 = (uint32_t)(32 * q + 16) << 16;
        // A block of this warp: rows 16q..16q+15, columns 32ch..32ch+31
        const bool a_zero = 16 * q + 15 < 32 * ch;      // entirely above the diagonal
        const bool a_full = 16 * q >= 32 * ch + 32;     // entirely below the diagonal
        const int hr0 = hi_row(r0), hr1 = hi_row(r1);
        // state S[i][j] held transposed: rows j = r0, r1; columns i = cbase + 8k + {0,1}
        float2 S0[4], S1[4];
        {
            const float* src = pseg > 0 ? seg.s_mid + ((size_t)bh * (seg.P - 1) + (pseg - 1)) * 4096
                                     : s_in ? s_in + (size_t)bh * 4096 : nullptr;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = cbase + 8 * k;
                S0[k] = src ? make_float2(src[i * 64 + r0], src[(i + 1) * 64 + r0]) : make_float2(0.f, 0.f);
                S1[k] = src ? make_float2(src[i * 64 + r1], src[(i + 1) * 64 + r1]) : make_float2(0.f, 0.f);
            }
            store_state(s.sb[0], S0, S1, r0, r1, ch, cb);   // S entering chunk 0, read by RO(0)
            if (a_zero) {                     // blocks of A that are always zero: once, here
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sts32(s.at, sw_off(hr0, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr0 + 8, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1 + 8, 4 * ch + k) + cb, 0u);
                }
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.s_ready[0]);
        }
        uint32_t up0[4] = {0u, 0u, 0u, 0u}, up1[4] = {0u, 0u, 0u, 0u};   // u' of the next output
        int n = 0;
        for (; n < NC; ++n) {
            const int pb = n & 1;
            // Finch-C2: u' of chunk n-1 is read from HBM now and used by output(n-1) below
            if (kC2 && n >= 1) load_uprime(uprime, n - 1, cseg, b, h, T, H, cbase, r0, r1, up0, up1);
            // ---- state(n): S <- gamma (S + U), U^T[j][i] = DU[j][i] + DU[j][64+i]
            {
                // gamma and bonus of chunk n reach us from prep through the chain prep's
                // release-arrive on prep_done -> the GU issuer's acquire -> its commit on gu_done
                const bool ok = wait_soft(s, &s.gu_done[pb], (uint32_t)((n >> 1) & 1), budget);
                // uniform over the epilogue: stop (hand-off) or abort
                if (named_bar_any(kBarEpi, kEpiThreads, !ok || ld_volatile(&s.abort) || ld_volatile(&s.stop_at) == n)) break;
            }
            ptx::tc_fence_after();
            {
                uint32_t ua[16], ub[16];
                tmem_ld16x4(tmem + lane_h0 + COL_DU + 128 * pb + 32 * ch, ua);
                tmem_ld16x4(tmem + lane_h0 + COL_DU + 128 * pb + 64 + 32 * ch, ub);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                mbar_arrive(&s.du_free[pb]);
                float2 gv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) gv[k] = *reinterpret_cast<const float2*>(&s.gamma[pb][cbase + 8 * k]);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 du0 = __fadd2_rn(lo_pair(ua, k), lo_pair(ub, k));
                    const float2 du1 = __fadd2_rn(hi_pair(ua, k), hi_pair(ub, k));
                    S0[k] = __fmul2_rn(gv[k], __fadd2_rn(S0[k], du0));
                    S1[k] = __fmul2_rn(gv[k], __fadd2_rn(S1[k], du1));
                }
            }
            if (n + 1 < NC) {
                // S_n feeds RO(n+1) from sb[(n+1) & 1], whose S_{n-2} RO(n-1) has read
                if (n >= 1) wait_soft(s, &s.s_free[(n - 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), budget);
                store_state(s.sb[(n + 1) & 1], S0, S1, r0, r1, ch, cb);
                ptx::fence_proxy_async_smem();
                mbar_arrive(&s.s_ready[(n + 1) & 1]);
            }
            // ---- output of chunk n-1 (its GA was issued at the end of the previous round)
            if (n >= 1)
                output_chunk<kC2>(s, n - 1, cseg, tmem, lane_h0, lane_h1, ch, cbase, r0, r1, b, h, T, H, y, y_raw,
                                  up0, up1, budget);
            // ---- A(n): masked scores with the bonus on the diagonal, hi / lo, for GA(n)
            wait_soft(s, &s.sc_done[pb], (uint32_t)((n >> 1) & 1), budget);
            ptx::tc_fence_after();
            if (!a_zero) {
                uint32_t p0[16], p1[16];
                tmem_ld16x4(tmem + lane_h0 + COL_SC + 64 * pb + 32 * ch, p0);
                tmem_ld16x4(tmem + lane_h1 + COL_SC + 64 * pb + 32 * ch, p1);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                mbar_arrive(&s.sc_free[pb]);
                const float b0 = kC2 ? 0.f : s.bonus[pb][r0], b1 = kC2 ? 0.f : s.bonus[pb][r1];
                // the A tile is free: GA(n-1) completed before output(n-1) read Y
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float2 a0 = rows_sum(p0, k), a1 = rows_sum(p1, k);
                    if (!a_full) {   // strictly causal scores, bonus on the diagonal
                        const int sx = cbase + 8 * k;
                        a0.x = sx < r0 ? a0.x : (sx == r0 ? b0 : 0.f);
                        a0.y = sx + 1 < r0 ? a0.y : (sx + 1 == r0 ? b0 : 0.f);
                        a1.x = sx < r1 ? a1.x : (sx == r1 ? b1 : 0.f);
                        a1.y = sx + 1 < r1 ? a1.y : (sx + 1 == r1 ? b1 : 0.f);
                    }
                    uint32_t hi, lo;
                    split2(a0, hi, lo);
                    sts32(s.at, sw_off(hr0, 4 * ch + k) + cb, hi);
                    sts32(s.at, sw_off(hr0 + 8, 4 * ch + k) + cb, lo);
                    split2(a1, hi, lo);
                    sts32(s.at, sw_off(hr1, 4 * ch + k) + cb, hi);
                    sts32(s.at, sw_off(hr1 + 8, 4 * ch + k) + cb, lo);
                }
            } else {
                ptx::tc_fence_before();
                mbar_arrive(&s.sc_free[pb]);
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.a_ready);
            mbar_arrive(&s.ep_free[pb]);      // gamma / bonus of parity pb read
        }
        // ---- leave: output of the last chunk done, final state (or the state entering the
        // chunk handed to the level kernel)
        if (!ld_volatile(&s.abort) && n >= 1) {
            if (kC2) load_uprime(uprime, n - 1, cseg, b, h, T, H, cbase, r0, r1, up0, up1);
            output_chunk<kC2>(s, n - 1, cseg, tmem, lane_h0, lane_h1, ch, cbase, r0, r1, b, h, T, H, y, y_raw,
                              up0, up1, budget);
        }
        const bool aborted = ld_volatile(&s.abort) != 0;
        if (!aborted) {
            const bool stopped = (n < NC);
            float* dst = stopped                       ? handoff_state + (size_t)unit * 4096
                         : (s_out && pseg == seg.P - 1) ? s_out + (size_t)bh * 4096
                                                     : nullptr;
            if (dst) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = cbase + 8 * k;
                    dst[i * 64 + r0] = S0[k].x;
                    dst[(i + 1) * 64 + r0] = S0[k].y;
                    dst[i * 64 + r1] = S1[k].x;
                    dst[(i + 1) * 64 + r1] = S1[k].y;
                }
            }
            if (tid == kEpiWarp0 * 32) handoff_chunk[unit] = stopped ? cseg + n : -1;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (s.abort && tid == 0) {
        atomicExch(status, 1);
        handoff_chunk[unit] = -1;
    }
    if (warp == kTmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

size_t fast_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_chunked_fast(const CUtensorMap* maps, const float* u, const float* s_in,
                                float* s_out, void* y, float* y_raw, int B, int T, int H,
                                Segments seg, Variant var, int* status, int* handoff_chunk,
                                float* handoff_state, long long budget, cudaStream_t st) {
    const size_t smem = fast_smem_bytes();
    auto kernel = var.uprime ? wkv6_fast_kernel<true> : wkv6_fast_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)(B * H * seg.P), kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], u, s_in, s_out, static_cast<__nv_bfloat16*>(y),
        y_raw, static_cast<const __nv_bfloat16*>(var.uprime), T, H, seg, status, handoff_chunk,
        handoff_state, budget, 4000000000LL);
    return cudaGetLastError();
}

}  // namespace goldwkv
