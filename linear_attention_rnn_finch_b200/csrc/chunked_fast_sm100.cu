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
// Precision.  Every operand that is rounded to bf16 -- Rt, Kh, S and A -- is split into
// hi = bf16(x) and lo = bf16(x - hi).  The lo parts cost no extra MMA instructions: hi and
// lo rows are stacked into M = 128 (rows 0-7 of every 16-row group hold hi parts of 8
// tokens, rows 8-15 the lo parts of the same tokens), and a 16x256b TMEM load hands each
// thread the hi and lo element of the same (token, column) in registers {0,1} / {2,3}, so
// the combination is one add in registers.  With all parts split the arithmetic is as
// accurate as fp32; the only bf16 rounding left is that of the output y.
//
// Per chunk three MMA groups (K = 64, four K16 instructions per chain):
//   G1: [Rt_hi ; Rt_lo] (M=128) x [S_hi^T ; Kh_hi]^T, then x [S_lo^T ; Kh_lo]^T accumulated
//       into the same columns (N=128) -> D1: columns 0..63 readout Rt . S, columns 64..127
//       intra-chunk scores Rt . Kh (hi and lo parts of S and Kh summed by the MMA)
//   GU: V^T (M=64) x [Kh_hi | Kh_lo] (N=128) -> DU = (Kh^T V)^T, the state increment
//   GA: [A_hi ; A_lo] (M=128) x V (N=64) -> DA, the intra-chunk output A . V
//
// Warp roles (448 threads): warp 0 TMA producer (3-stage ring of r, k, v, omega tiles);
// warp 1 MMA issuer (and TMEM owner); warps 2-5 prep (log-decay scan, Rt / Kh operands,
// bonus, gamma, range test); warps 6-13 epilogue (state update, assembly of A, output).
// Handshakes are mbarriers; every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

constexpr int C = 64;
constexpr int kStages = 3;
constexpr int kTile = 64 * 64 * 2;            // 64 rows x 128 B
constexpr int kThreads = 448;
constexpr int kPrepWarp0 = 2, kEpiWarp0 = 6;
constexpr int kEpiThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_D1 = 0, COL_DU = 128, COL_DA = 256;
// log2 of the largest factor exp(-L_s) allowed: ln range 60 -> log2 range 86.56
constexpr float kMaxLog2Range = 86.5617f;
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t IDESC_G1 = ptx::idesc_bf16(128, 128, 0, 0);
constexpr uint32_t IDESC_GU = ptx::idesc_bf16(64, 128, 1, 1);
constexpr uint32_t IDESC_GA = ptx::idesc_bf16(128, 64, 0, 1);

struct __align__(1024) Smem {
    uint8_t in[kStages][4][kTile];   // r, k, v, omega tiles (TMA, 128B swizzle)
    uint8_t bblk[2][4][kTile];       // per parity: S_hi^T, Kh_hi, S_lo^T, Kh_lo (G1 operand B)
    uint8_t rt[2][2 * kTile];        // per parity: Rt hi/lo, 128 stacked rows (G1 operand A)
    uint8_t at[2 * kTile];           // A hi/lo, 128 stacked rows (GA operand A)
    uint8_t ystage[kTile];           // y tile for the TMA store
    float qtot[4][64];               // prep: per-quarter sums of log2 w
    float gamma[2][64];
    float bonus[2][64];
    int unsafe[2];
    uint64_t full[kStages], empty[kStages];
    uint64_t prep_done[2], op_free[2];
    uint64_t g1_done, ga_done, epi_mid, epi_end, s_init;
    uint32_t tmem_base;
    int abort;
    int stop_at;                     // chunk at which this (b,h) leaves for the level kernel
};

__device__ __forceinline__ uint32_t sw_off(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
// stacked hi/lo row of token t: hi parts in rows 0-7 of each 16-row group, lo in rows 8-15
__device__ __forceinline__ int hi_row(int t) { return 32 * (t >> 4) + 16 * ((t >> 3) & 1) + (t & 7); }

// bf16x2 of (a, b): a in the low half (lower address), b in the high half
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// hi = bf16(x), lo = bf16(x - hi) for a pair: two conversions and one packed subtract
__device__ __forceinline__ void split2(float2 x, uint32_t& hi, uint32_t& lo) {
    hi = pack2(x.x, x.y);
    const float2 d = __fadd2_rn(x, make_float2(-__uint_as_float(hi << 16),
                                               -__uint_as_float(hi & 0xFFFF0000u)));
    lo = pack2(d.x, d.y);
}
__device__ __forceinline__ void sts32(uint8_t* base, uint32_t off, uint32_t v) {
    *reinterpret_cast<uint32_t*>(base + off) = v;
}
__device__ __forceinline__ uint32_t lds32(const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(base + off);
}
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 16 lanes x 256 bits x 4: thread l gets lanes base + l/4 (regs 4k, 4k+1) and
// base + 8 + l/4 (regs 4k+2, 4k+3), columns col + 8k + 2(l%4) + {0,1}, k = 0..3.
__device__ __forceinline__ void tmem_ld16x4(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// barrier over `nthreads` threads that also ORs a predicate across them (uniform decision)
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_addr(bar)) : "memory");
}

__device__ __forceinline__ int ld_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

__global__ void __launch_bounds__(kThreads, 1)
wkv6_fast_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ u,
                 const float* s_in, float* s_out, float* __restrict__ y_raw, int T, int H,
                 int* status, int* handoff_chunk, float* handoff_state, long long budget,
                 long long drain_budget) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x, b = bh / H, h = bh - (bh / H) * H;
    const int NC = (T + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&s.full[i], 1);
            ptx::mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.prep_done[i], 128);
            ptx::mbar_init(&s.op_free[i], 1);
        }
        ptx::mbar_init(&s.g1_done, 1);
        ptx::mbar_init(&s.ga_done, 1);
        ptx::mbar_init(&s.epi_mid, kEpiThreads);
        ptx::mbar_init(&s.epi_end, kEpiThreads);
        ptx::mbar_init(&s.s_init, kEpiThreads);
        ptx::fence_mbar_init();
        s.abort = 0;
        s.stop_at = -1;
    }
    if (warp == 1) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tensormap(&tm_r);
            ptx::prefetch_tensormap(&tm_k);
            ptx::prefetch_tensormap(&tm_v);
            ptx::prefetch_tensormap(&tm_w);
            int last[kStages] = {-1, -1, -1};
            for (int n = 0; n < NC; ++n) {
                const int st = n % kStages;
                if (n >= kStages) {
                    // wait for the stage to be released; give up if this head stopped
                    const uint32_t par = (uint32_t)(((n - kStages) / kStages) & 1);
                    bool ok = false;
                    const long long t0 = clock64();
                    for (;;) {
                        if (ptx::mbar_try_wait(&s.empty[st], par)) { ok = true; break; }
                        if (ld_volatile(&s.stop_at) >= 0 || ld_volatile(&s.abort)) break;
                        if (clock64() - t0 > budget) { s.abort = 1; break; }
                    }
                    if (!ok) break;
                }
                ptx::mbar_arrive_expect_tx(&s.full[st], 4 * kTile);
                const int t0 = n * C;
                ptx::tma_load_4d(s.in[st][0], &tm_r, &s.full[st], 0, h, t0, b);
                ptx::tma_load_4d(s.in[st][1], &tm_k, &s.full[st], 0, h, t0, b);
                ptx::tma_load_4d(s.in[st][2], &tm_v, &s.full[st], 0, h, t0, b);
                ptx::tma_load_4d(s.in[st][3], &tm_w, &s.full[st], 0, h, t0, b);
                last[st] = n;
            }
            // every issued copy must land before the CTA may exit
            for (int st = 0; st < kStages; ++st)
                if (last[st] >= 0)
                    ptx::mbar_wait(&s.full[st], (uint32_t)((last[st] / kStages) & 1), drain_budget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int last_g1 = -1, last_ga = -1;
            for (int n = 0; n < NC; ++n) {
                const int pb = n & 1, st = n % kStages;
                if (!ptx::mbar_wait(&s.prep_done[pb], (uint32_t)((n >> 1) & 1), budget)) { s.abort = 1; break; }
                if (s.unsafe[pb]) {          // hand this (b,h) to the level kernel from chunk n
                    s.stop_at = n;
                    mbar_arrive(&s.g1_done);  // wakes the epilogue, which saves the state
                    break;
                }
                // D1 / DU free and S_n written: the epilogue finished state + assembly of n-1
                // (for n = 0: the initial state is in shared memory)
                if (n == 0 && !ptx::mbar_wait(&s.s_init, 0, budget)) { s.abort = 1; break; }
                if (n > 0 && !ptx::mbar_wait(&s.epi_mid, (uint32_t)((n - 1) & 1), budget)) { s.abort = 1; break; }
                ptx::tc_fence_after();
                const uint32_t v_tile = ptx::smem_addr(s.in[st][2]);
                const uint32_t bhi = ptx::smem_addr(s.bblk[pb][0]);   // [S_hi^T ; Kh_hi]
                const uint32_t blo = ptx::smem_addr(s.bblk[pb][2]);   // [S_lo^T ; Kh_lo]
                const uint32_t kh = ptx::smem_addr(s.bblk[pb][1]);
                const uint32_t rt = ptx::smem_addr(s.rt[pb]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // GU: V^T x [Kh_hi | Kh_lo] (N atoms 16 KB apart)
                    ptx::mma_bf16(tmem + COL_DU, ptx::desc_sw128(v_tile + 2048 * kq, 1024),
                                  ptx::desc_sw128(kh + 2048 * kq, 2 * kTile), IDESC_GU, kq > 0);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   // G1: [Rt] x [S_hi^T ; Kh_hi]
                    ptx::mma_bf16(tmem + COL_D1, ptx::desc_kmajor(rt + 32 * kq),
                                  ptx::desc_kmajor(bhi + 32 * kq), IDESC_G1, kq > 0);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)   //   + [Rt] x [S_lo^T ; Kh_lo]
                    ptx::mma_bf16(tmem + COL_D1, ptx::desc_kmajor(rt + 32 * kq),
                                  ptx::desc_kmajor(blo + 32 * kq), IDESC_G1, 1);
                ptx::mma_commit(&s.g1_done);
                last_g1 = n;
                // GA needs A (assembly of n) and DA free (output of n-1 read)
                if (!ptx::mbar_wait(&s.epi_mid, (uint32_t)(n & 1), budget)) { s.abort = 1; break; }
                if (n > 0 && !ptx::mbar_wait(&s.epi_end, (uint32_t)((n - 1) & 1), budget)) { s.abort = 1; break; }
                ptx::tc_fence_after();
                const uint32_t at = ptx::smem_addr(s.at);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    ptx::mma_bf16(tmem + COL_DA, ptx::desc_kmajor(at + 32 * kq),
                                  ptx::desc_mnmajor(v_tile + 2048 * kq), IDESC_GA, kq > 0);
                ptx::mma_commit(&s.ga_done);
                ptx::mma_commit(&s.empty[st]);     // stage read by GU / GA (prep read it before)
                ptx::mma_commit(&s.op_free[pb]);   // Rt / Kh / gamma / bonus of parity pb
                last_ga = n;
            }
            // drain: our own tensor-core work must be complete before TMEM is freed
            if (last_g1 >= 0) ptx::mbar_wait(&s.g1_done, (uint32_t)(last_g1 & 1), drain_budget);
            if (last_ga >= 0) ptx::mbar_wait(&s.ga_done, (uint32_t)(last_ga & 1), drain_budget);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ prep (4 warps)
        // lane = channel pair (2l, 2l+1), warp = token quarter (16 tokens); log2 units
        const int qw = warp - kPrepWarp0;
        const int c0 = 2 * lane;
        const float2 uu = make_float2(u[h * 64 + c0], u[h * 64 + c0 + 1]);
        const int chunk = lane >> 2;          // 16-byte chunk holding channels c0, c0+1
        const uint32_t cbyte = (uint32_t)(lane & 3) * 4;
        const float2 l2e = make_float2(kLog2e, kLog2e);
        const float2 nl2e = make_float2(-kLog2e, -kLog2e);
        for (int n = 0; n < NC; ++n) {
            const int pb = n & 1, st = n % kStages;
            const int valid = min(C, T - n * C);
            bool bad = !ptx::mbar_wait(&s.full[st], (uint32_t)((n / kStages) & 1), budget);
            if (n >= 2) bad |= !ptx::mbar_wait(&s.op_free[pb], (uint32_t)(((n - 2) >> 1) & 1), budget);
            if (bad) s.abort = 1;
            if (named_bar_any(1, 128, bad || ld_volatile(&s.abort))) break;   // uniform over prep
            const uint8_t* r_tile = s.in[st][0];
            const uint8_t* k_tile = s.in[st][1];
            const uint8_t* w_tile = s.in[st][3];
            // pass 1: local inclusive prefix of log2 w = -exp(omega) log2(e)
            float2 L[16];
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int t = 16 * qw + p;
                const float2 om = __fmul2_rn(unpack2(lds32(w_tile, sw_off(t, chunk) + cbyte)), l2e);
                float2 e = make_float2(fast_exp2(om.x), fast_exp2(om.y));
                if (t >= valid) e = make_float2(0.f, 0.f);
                acc = __ffma2_rn(e, nl2e, acc);
                L[p] = acc;
            }
            s.qtot[qw][c0] = acc.x;
            s.qtot[qw][c0 + 1] = acc.y;
            named_bar(1, 128);
            float2 off = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float2 qv = make_float2(s.qtot[w][c0], s.qtot[w][c0 + 1]);
                if (w < qw) off = __fadd2_rn(off, qv);
                tot = __fadd2_rn(tot, qv);
            }
            const bool ok = __all_sync(0xffffffffu, (tot.x >= -kMaxLog2Range) && (tot.y >= -kMaxLog2Range));
            if (!ok) {
                if (qw == 0 && lane == 0) s.unsafe[pb] = 1;
                named_bar(1, 128);           // qtot is reused by the next chunk
                mbar_arrive(&s.prep_done[pb]);
                break;                        // this (b,h) continues in the level kernel
            }
            // pass 2: Rt = r 2^(L_{t-1}), Kh = k 2^(-L_t) as bf16 hi / lo; bonus partials
            uint8_t* rt = s.rt[pb];
            uint8_t* kh_hi = s.bblk[pb][1];
            uint8_t* kh_lo = s.bblk[pb][3];
            float bon[16];
            float2 fr = make_float2(fast_exp2(off.x), fast_exp2(off.y));   // 2^(L_{t-1})
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int t = 16 * qw + p;
                const uint32_t o = sw_off(t, chunk) + cbyte;
                const float2 rr = unpack2(lds32(r_tile, o));
                const float2 kk = unpack2(lds32(k_tile, o));
                const float2 li = __fadd2_rn(off, L[p]);
                const float2 fk = make_float2(fast_exp2(-li.x), fast_exp2(-li.y));
                uint32_t hi, lo;
                split2(__fmul2_rn(rr, fr), hi, lo);
                const int hr = hi_row(t);
                const uint32_t cb = (uint32_t)(chunk ^ (t & 7)) << 4;
                sts32(rt, (uint32_t)hr * 128 + cb + cbyte, hi);
                sts32(rt, (uint32_t)(hr + 8) * 128 + cb + cbyte, lo);
                split2(__fmul2_rn(kk, fk), hi, lo);
                sts32(kh_hi, o, hi);
                sts32(kh_lo, o, lo);
                const float2 ru = __fmul2_rn(rr, uu);
                bon[p] = fmaf(ru.x, kk.x, ru.y * kk.y);
                if (p < 15) fr = make_float2(fast_exp2(li.x), fast_exp2(li.y));
            }
            // bonus: reduce the 16 per-token partials over the 32 lanes (reduce-scatter)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const bool up = lane & 16;
                const float send = up ? bon[i] : bon[i + 8];
                const float keep = up ? bon[i + 8] : bon[i];
                bon[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool up = lane & 8;
                const float send = up ? bon[i] : bon[i + 4];
                const float keep = up ? bon[i + 4] : bon[i];
                bon[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const bool up = lane & 4;
                const float send = up ? bon[i] : bon[i + 2];
                const float keep = up ? bon[i + 2] : bon[i];
                bon[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            {
                const bool up = lane & 2;
                const float send = up ? bon[0] : bon[1];
                const float keep = up ? bon[1] : bon[0];
                bon[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            bon[0] += __shfl_xor_sync(0xffffffffu, bon[0], 1);
            if ((lane & 1) == 0) {
                const int p = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                              ((lane >> 1) & 1);
                s.bonus[pb][16 * qw + p] = bon[0];
            }
            if (qw == 0) {
                s.gamma[pb][c0] = fast_exp2(tot.x);
                s.gamma[pb][c0 + 1] = fast_exp2(tot.y);
                if (lane == 0) s.unsafe[pb] = 0;
            }
            ptx::fence_proxy_async_smem();
            named_bar(1, 128);               // qtot reads done before the next chunk writes it
            mbar_arrive(&s.prep_done[pb]);
        }
    } else {
        // ------------------------------------------------------------ epilogue (8 warps)
        // warp (q, ch): TMEM sub-partition q, columns 32ch .. 32ch+31 of each 64-wide block.
        // Thread: token / state rows r0 = 16q + l/4 and r1 = r0 + 8; column pairs
        // cbase + 8k + {0,1}, k = 0..3.
        const int q = warp & 3;
        const int ch = (warp - kEpiWarp0) >> 2;
        const int et = tid - kEpiWarp0 * 32;  // 0 .. 255
        const int r0 = 16 * q + (lane >> 2), r1 = r0 + 8;
        const int cbase = 32 * ch + 2 * (lane & 3);
        const uint32_t cb = (uint32_t)(lane & 3) * 4;
        const uint32_t lane_m64 = (uint32_t)(32 * q) << 16;
        const uint32_t lane_h0 = (uint32_t)(32 * q) << 16, lane_h1 = (uint32_t)(32 * q + 16) << 16;
        // A block of this warp: rows 16q..16q+15, columns 32ch..32ch+31
        const bool a_zero = 16 * q + 15 < 32 * ch;      // entirely above the diagonal
        const bool a_full = 16 * q >= 32 * ch + 32;     // entirely below the diagonal
        const int hr0 = hi_row(r0), hr1 = hi_row(r1);
        // state S[i][j] held transposed: rows j = r0, r1; columns i = cbase + 8k + {0,1}
        float2 S0[4], S1[4];
        {
            const float* src = s_in ? s_in + (size_t)bh * 4096 : nullptr;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = cbase + 8 * k;
                S0[k] = src ? make_float2(src[i * 64 + r0], src[(i + 1) * 64 + r0]) : make_float2(0.f, 0.f);
                S1[k] = src ? make_float2(src[i * 64 + r1], src[(i + 1) * 64 + r1]) : make_float2(0.f, 0.f);
            }
            // S_0 into parity 0: S_hi^T (tile 0) / S_lo^T (tile 2), rows j, K index i
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t hi, lo;
                split2(S0[k], hi, lo);
                sts32(s.bblk[0][0], sw_off(r0, 4 * ch + k) + cb, hi);
                sts32(s.bblk[0][2], sw_off(r0, 4 * ch + k) + cb, lo);
                split2(S1[k], hi, lo);
                sts32(s.bblk[0][0], sw_off(r1, 4 * ch + k) + cb, hi);
                sts32(s.bblk[0][2], sw_off(r1, 4 * ch + k) + cb, lo);
            }
            // blocks of A that are always zero are written once here
            if (a_zero) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sts32(s.at, sw_off(hr0, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr0 + 8, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1, 4 * ch + k) + cb, 0u);
                    sts32(s.at, sw_off(hr1 + 8, 4 * ch + k) + cb, 0u);
                }
            }
            ptx::fence_proxy_async_smem();
            mbar_arrive(&s.s_init);
        }
        // sum of the hi row (regs 4k, 4k+1) and lo row (regs 4k+2, 4k+3) of a 16x256b load
        auto rows_sum = [](const uint32_t (&v)[16], int k) {
            return __fadd2_rn(make_float2(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1])),
                              make_float2(__uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3])));
        };
        int n = 0;
        for (; n < NC; ++n) {
            const int pb = n & 1;
            const int valid = min(C, T - n * C);
            {
                bool bad = !ptx::mbar_wait(&s.g1_done, (uint32_t)(n & 1), budget);
                // gamma / bonus of this chunk were written by prep before prep_done
                if (!bad && ld_volatile(&s.stop_at) != n)
                    bad = !ptx::mbar_wait(&s.prep_done[pb], (uint32_t)((n >> 1) & 1), budget);
                if (bad) s.abort = 1;
                // uniform over the epilogue group: stop (hand-off) or abort
                if (named_bar_any(3, kEpiThreads, bad || ld_volatile(&s.abort) || ld_volatile(&s.stop_at) == n)) break;
            }
            ptx::tc_fence_after();
            // ---- state: S <- gamma (S + U), U^T[j][i] = DU[j][i] + DU[j][64+i]
            {
                uint32_t ua[16], ub[16];
                tmem_ld16x4(tmem + lane_m64 + COL_DU + 32 * ch, ua);
                tmem_ld16x4(tmem + lane_m64 + COL_DU + 64 + 32 * ch, ub);
                ptx::tmem_wait_ld();
                uint8_t* sh = s.bblk[pb ^ 1][0];
                uint8_t* sl = s.bblk[pb ^ 1][2];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 g = *reinterpret_cast<const float2*>(&s.gamma[pb][cbase + 8 * k]);
                    const float2 du0 = __fadd2_rn(make_float2(__uint_as_float(ua[4 * k]), __uint_as_float(ua[4 * k + 1])),
                                                  make_float2(__uint_as_float(ub[4 * k]), __uint_as_float(ub[4 * k + 1])));
                    const float2 du1 = __fadd2_rn(make_float2(__uint_as_float(ua[4 * k + 2]), __uint_as_float(ua[4 * k + 3])),
                                                  make_float2(__uint_as_float(ub[4 * k + 2]), __uint_as_float(ub[4 * k + 3])));
                    S0[k] = __fmul2_rn(g, __fadd2_rn(S0[k], du0));
                    S1[k] = __fmul2_rn(g, __fadd2_rn(S1[k], du1));
                    uint32_t hi, lo;
                    split2(S0[k], hi, lo);
                    sts32(sh, sw_off(r0, 4 * ch + k) + cb, hi);
                    sts32(sl, sw_off(r0, 4 * ch + k) + cb, lo);
                    split2(S1[k], hi, lo);
                    sts32(sh, sw_off(r1, 4 * ch + k) + cb, hi);
                    sts32(sl, sw_off(r1, 4 * ch + k) + cb, lo);
                }
            }
            // ---- readout part Yi (kept in registers) and scores A -> A_hi / A_lo tiles
            float2 Y0[4], Y1[4];
            {
                uint32_t p0[16], p1[16];
                tmem_ld16x4(tmem + lane_h0 + COL_D1 + 32 * ch, p0);
                tmem_ld16x4(tmem + lane_h1 + COL_D1 + 32 * ch, p1);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    Y0[k] = rows_sum(p0, k);
                    Y1[k] = rows_sum(p1, k);
                }
            }
            if (!a_zero) {
                uint32_t p0[16], p1[16];
                tmem_ld16x4(tmem + lane_h0 + COL_D1 + 64 + 32 * ch, p0);
                tmem_ld16x4(tmem + lane_h1 + COL_D1 + 64 + 32 * ch, p1);
                ptx::tmem_wait_ld();
                const float b0 = s.bonus[pb][r0], b1 = s.bonus[pb][r1];
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
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            mbar_arrive(&s.epi_mid);
            // ---- output: y = Yi + A.V
            {
                const bool bad = !ptx::mbar_wait(&s.ga_done, (uint32_t)(n & 1), budget);
                if (bad) s.abort = 1;
                if (named_bar_any(3, kEpiThreads, bad || ld_volatile(&s.abort))) break;
            }
            ptx::tc_fence_after();
            {
                uint32_t d0[16], d1[16];
                tmem_ld16x4(tmem + lane_h0 + COL_DA + 32 * ch, d0);
                tmem_ld16x4(tmem + lane_h1 + COL_DA + 32 * ch, d1);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    Y0[k] = __fadd2_rn(Y0[k], rows_sum(d0, k));
                    Y1[k] = __fadd2_rn(Y1[k], rows_sum(d1, k));
                }
            }
            ptx::tc_fence_before();
            mbar_arrive(&s.epi_end);    // DA read: GA of the next chunk may overwrite it
            if (y_raw != nullptr) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int j = cbase + 8 * k;
                    if (r0 < valid)
                        *reinterpret_cast<float2*>(y_raw + (((size_t)b * T + n * C + r0) * H + h) * 64 + j) = Y0[k];
                    if (r1 < valid)
                        *reinterpret_cast<float2*>(y_raw + (((size_t)b * T + n * C + r1) * H + h) * 64 + j) = Y1[k];
                }
            } else {
                // the previous chunk's store must have read the staging tile
                if (et == 0) ptx::bulk_wait_read<0>();
                named_bar(2, kEpiThreads);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    sts32(s.ystage, sw_off(r0, 4 * ch + k) + cb, pack2(Y0[k].x, Y0[k].y));
                    sts32(s.ystage, sw_off(r1, 4 * ch + k) + cb, pack2(Y1[k].x, Y1[k].y));
                }
                ptx::fence_proxy_async_smem();
                named_bar(2, kEpiThreads);
                if (et == 0) {
                    ptx::tma_store_4d(&tm_y, s.ystage, 0, h, n * C, b);
                    ptx::bulk_commit();
                }
            }
        }
        // ---- leave: final state, or the state entering the chunk handed to the level kernel
        const bool aborted = ld_volatile(&s.abort) != 0;
        if (!aborted) {
            const bool stopped = (n < NC);
            float* dst = stopped ? handoff_state + (size_t)bh * 4096 : s_out ? s_out + (size_t)bh * 4096 : nullptr;
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
            if (et == 0) handoff_chunk[bh] = stopped ? n : -1;
        }
        if (et == 0) ptx::bulk_wait<0>();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (s.abort && tid == 0) {
        atomicExch(status, 1);
        handoff_chunk[bh] = -1;
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

size_t fast_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_chunked_fast(const CUtensorMap* maps, const float* u, const float* s_in,
                                float* s_out, float* y_raw, int B, int T, int H, int* status,
                                int* handoff_chunk, float* handoff_state, long long budget,
                                cudaStream_t st) {
    const size_t smem = fast_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(wkv6_fast_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    wkv6_fast_kernel<<<(unsigned)(B * H), kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], u, s_in, s_out, y_raw, T, H, status,
        handoff_chunk, handoff_state, budget, 4000000000LL);
    return cudaGetLastError();
}

}  // namespace goldwkv
