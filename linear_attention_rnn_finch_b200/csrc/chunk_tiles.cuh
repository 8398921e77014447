// Device helpers shared by the tcgen05 chunk kernels: 128B-swizzled tile addressing, bf16
// pair packing and hi/lo splitting, 16x256b TMEM loads, named barriers and bounded
// mbarrier waits.  Include only from CUDA sources compiled for sm_100a.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace goldwkv {
namespace tiles {

constexpr int kTile = 64 * 64 * 2;   // one 64-row x 128-byte tile (64 x 64 bf16)

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
// The same shape repeated 8 times: columns col + 8k + 2(l%4) + {0,1}, k = 0..7.
__device__ __forceinline__ void tmem_ld16x8(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
}
// the (hi row + lo row) pair k of a 16x256b load: registers 4k, 4k+1 plus 4k+2, 4k+3
template <int N>
__device__ __forceinline__ float2 rows_sum(const uint32_t (&v)[N], int k) {
    return __fadd2_rn(make_float2(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1])),
                      make_float2(__uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3])));
}
template <int N>
__device__ __forceinline__ float2 lo_pair(const uint32_t (&v)[N], int k) {
    return make_float2(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]));
}
template <int N>
__device__ __forceinline__ float2 hi_pair(const uint32_t (&v)[N], int k) {
    return make_float2(__uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
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

// 1 - exp(-x) for x = exp(omega) >= 0 (the Finch-C2 key factor 1 - w), without the
// cancellation of 1 - w for small x: below 1/4 the series x (1 - x/2 (1 - x/3 (1 - x/4
// (1 - x/5)))), whose first omitted term is x^6/720 (relative error < 1.5e-6 there);
// from 1/4 up, 1 - 2^(-x log2 e) directly (w <= 0.78, so the subtraction loses < 3 bits).
__device__ __forceinline__ float2 one_minus_exp_neg2(float2 x) {
    const float2 one = make_float2(1.f, 1.f);
    float2 p = __ffma2_rn(x, make_float2(-0.2f, -0.2f), one);
    p = __ffma2_rn(__fmul2_rn(x, make_float2(-0.25f, -0.25f)), p, one);
    p = __ffma2_rn(__fmul2_rn(x, make_float2(-1.f / 3.f, -1.f / 3.f)), p, one);
    p = __ffma2_rn(__fmul2_rn(x, make_float2(-0.5f, -0.5f)), p, one);
    p = __fmul2_rn(x, p);
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 d = make_float2(1.f - fast_exp2(x.x * kNegLog2e), 1.f - fast_exp2(x.y * kNegLog2e));
    return make_float2(x.x < 0.25f ? p.x : d.x, x.y < 0.25f ? p.y : d.y);
}

// How long one try_wait of a bounded wait may sleep before the thread looks at the CTA's
// abort / hand-over words and its budget again (nanoseconds; 0: poll without sleeping).  A
// hand-over wakes the threads still waiting for chunks that will not come within about
// this time.
#ifndef GW_WAIT_SLEEP_NS
#define GW_WAIT_SLEEP_NS 2000
#endif
constexpr uint32_t kWaitSleepNs = GW_WAIT_SLEEP_NS;

// The dynamic shared memory rounded up to a 1024-byte boundary (the 128B-swizzle atom),
// derived from the __shared__ array by pointer arithmetic only: the compiler then still
// knows every access through it is to shared memory (32-bit addressed LDS / STS, not
// generic loads and stores).
template <class T>
__device__ __forceinline__ T& smem_aligned(uint8_t* raw) {
    const uint32_t pad = (1024u - (ptx::smem_addr(raw) & 1023u)) & 1023u;
    return *reinterpret_cast<T*>(raw + pad);
}

// Bounded wait on an mbarrier phase.  `s` is the CTA's shared state with `abort` and
// `stop_at` words: the wait gives up early once the CTA has aborted, and on expiry it aborts
// the CTA.
// Returns false if the caller should treat its data as invalid (abort).
// With stop_chunk >= 0, also gives up (without aborting) once this (b,h) has been handed
// over at or before chunk stop_chunk (stop_at <= stop_chunk).
template <class Sm>
__device__ __forceinline__ bool wait_soft(Sm& s, uint64_t* bar, uint32_t parity, long long budget,
                                          int stop_chunk = -1) {
    if (ptx::mbar_test_wait(bar, parity)) return true;
    if (stop_chunk >= 0 && ld_volatile(&s.stop_at) <= stop_chunk) return false;
    if (budget <= 0) {
        s.abort = 1;
        return false;
    }
    const long long t0 = clock64();
    for (;;) {
#ifdef GW_CONTROL_SPIN
        const bool sleep = kWaitSleepNs > 0 && threadIdx.x >= 96;
#else
        const bool sleep = kWaitSleepNs > 0;
#endif
        if (sleep ? ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)
                  : ptx::mbar_try_wait(bar, parity))
            return true;
        if (ld_volatile(&s.abort)) return false;
        if (stop_chunk >= 0 && ld_volatile(&s.stop_at) <= stop_chunk) return false;
        if (clock64() - t0 > budget) {
            s.abort = 1;
            return false;
        }
    }
}


}  // namespace tiles
}  // namespace goldwkv
