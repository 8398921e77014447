// Chunked WKV6 prefill on sm_100a: TMA-fed tcgen05 tensor-core contractions.
//
// What is computed (GoldFinch review page, section 3.4, "Recurrent state update and
// output" and "Data-dependent decay"): per (b,h) with D = 64,
//     y_t = r_t . (diag(u) k_t^T v_t + S_{t-1}),   S_t = diag(w_t) S_{t-1} + k_t^T v_t,
//     w_t = exp(-exp(omega_t)).
// The page's pre-fill runs the recurrence "in parallel chunks" (section 3.4, "Training and
// Inference Procedures"); this kernel is that chunked form.  For a chunk of C = 64 tokens
// with incoming state S (rows i: key/decay channels, columns j: value channels):
//
//   y_t   = Rt_t . S  +  sum_{s<t} A[t][s] v_s  +  A[t][t] v_t
//   S_out = diag(gamma) S + Kt^T V
// with  Rt_t = r_t * prod_{tau<t} w_tau,  Kt_s = k_s * prod_{tau>s} w_tau,
//       gamma = prod_{tau<C} w_tau,  A[t][t] = sum_i r_t[i] u[i] k_t[i]  (the bonus),
//       A[t][s] = sum_i r_t[i] k_s[i] prod_{s<tau<t} w_tau[i]   (s < t).
//
// Overflow-free decay factorisation of A.  Every decay factor is a product of w's over a
// range, i.e. <= 1.  Split the pairs (t, s), s < t, by the highest bit in which t and s
// differ, l in 0..5: both lie in one 2^(l+1)-aligned block, t in its upper 2^l half and s
// in the lower half, so
//     prod_{s<tau<t} w = [prod of w from the start of t's 2^l block to t-1]
//                      * [prod of w from s+1 to the end of s's 2^l block].
// With Q^l_t = r_t * (first bracket) and K^l_s = k_s * (second bracket) -- both <= |r|, |k|
// -- the pairs of level l are entries of the product Q^l (K^l)^T.  Level 0 needs no decay
// at all (Q^0 = r, K^0 = k: the raw TMA tiles).  Each level is one 64x64x64 tcgen05 MMA
// into its own TMEM accumulator; A is assembled by picking, for every (t, s), the entry of
// its level.  No exponential of a positive number is ever formed, so nothing overflows
// for any decay, and no clamp is needed.
//
// Precision: operands are bf16 with fp32 accumulation.  S and A, whose rounding would sit
// directly on y, are split into bf16 hi + lo parts (two MMAs each); the fp32 state chain
// S <- gamma*S + U stays in registers across chunks.
//
// Schedule (one CTA per (b,h), 256 threads, chunks in order, all warps in lockstep):
//   TMA loads of r, k, v, omega run two chunks ahead (2-stage ring, mbarrier tx-count);
//   prep    : warp = 8 channels, lane = 2 tokens; w, block products (shuffle butterfly),
//             operands Q^1..5, K^1..5, Rt, Kt^T written to 128B-swizzled smem;
//   MMA 1   : U = Kt^T V, Y = Rt S_hi + Rt S_lo (thread 0 issues, commit), then L^0..L^5
//             (commit);
//   state   : S <- gamma S + U in registers; S_hi/S_lo for the next chunk (once U and Y are
//             done, while the level products run);
//   assemble: A from the level accumulators, hi/lo to smem;
//   MMA 2   : Y += A_hi V + A_lo V;
//   epilogue: Y -> bf16 -> smem -> TMA store (double-buffered), or fp32 rows for the
//             LayerNorm (y_raw).
// LayerNorm over a token's H heads (the page's final output) can run in the same launch:
// extra CTAs, and the CTAs of units the fast kernel already finished, normalise 64-token
// blocks of a batch row once every head has published them (ln_blocks below; a cooperative
// launch keeps them co-resident with the units they wait for).
// An M=64 accumulator occupies lanes 0..15 of TMEM sub-partition q for rows 16q..16q+15,
// so warp w reads rows 16(w%4)..+15, columns split between warps w and w+4.  The state
// chain and the epilogue read them with a two-half load (lanes 16..31 of the warp get the
// same rows' next 16 columns): every lane holds a row, 16 columns; so does A's assembly.
//
// Every mbarrier wait is bounded (spin budget in SM cycles); on expiry the CTA records
// an error word, drains its in-flight copies and MMAs with a second bounded wait, frees
// its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <limits.h>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

constexpr int C = 64;                 // tokens per chunk
constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr int kTile = 64 * 64 * 2;    // one 64 x 64 bf16 tile, bytes
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_L0 = 0;        // level accumulators at 64*l
constexpr uint32_t COL_U = 384;
constexpr uint32_t COL_Y = 448;
constexpr uint32_t IDESC_KK = ptx::idesc_bf16(64, 64, 0, 0);
constexpr uint32_t IDESC_KM = ptx::idesc_bf16(64, 64, 0, 1);

struct __align__(1024) Smem {
    uint8_t in[kStages][4][kTile];   // r, k, v, omega tiles per stage (TMA, 128B swizzle)
    uint8_t q[5][kTile];             // Q^1..Q^5; q[0], q[1] are reused for A_hi, A_lo
    uint8_t kk[5][kTile];            // K^1..K^5
    uint8_t rt[kTile];               // Rt  [t][i]
    uint8_t ktT[kTile];              // Kt^T [i][s]
    uint8_t s_hi[kTile];             // S as bf16 [i][j], high part
    uint8_t s_lo[kTile];             // low part
    uint8_t ystage[2][kTile];        // y tiles for the TMA store
    float u[64];
    float gamma[64];
    float bonus_part[8][64];         // per channel group partial of sum_i r u k
    uint64_t full[kStages];
    uint64_t mma1u, mma1, mma2;   // MMA 1's U and Y products; all of MMA 1; MMA 2
    uint32_t tmem_base;
    int abort;
    int ln_go;                       // LayerNorm CTAs: every head of the block is stored
    int ln_rb;                       // LayerNorm CTAs: the block taken
    float2 gn_mom[2][64];            // GroupNorm stage: (mean, M2) of each row's two halves
};

// byte offset of element (row, col) in a 64 x 64 bf16 tile with 128-byte rows, swizzled
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

// hi = bf16(x), lo = bf16(x - hi): x ~= hi + lo to about 16 significant bits
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

__device__ __forceinline__ void st_shared_v4(uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One warp: LayerNorm of a row of nf4 16-byte pieces (nf4 <= 512, i.e. H <= 32 heads) read
// from L2 (the rows were written by other SMs during this launch), bf16 out.  The fp32 row
// is scratch nobody reads again: once it is in registers its 128-byte L2 lines are dropped
// (discard.global.L2: no write-back), so rows read soon after they were written never
// reach DRAM.  Only for a 128-byte-aligned row (the instruction's requirement).
__device__ __forceinline__ void ln_row_warp(const float* row, __nv_bfloat16* orow,
                                            const float* gamma, const float* beta, float eps,
                                            int nf4, int lane) {
    float4 v[16];
    float sm = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const int i = lane + 32 * m;
        v[m] = i < nf4 ? __ldcg(reinterpret_cast<const float4*>(row) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        sm += (v[m].x + v[m].y) + (v[m].z + v[m].w);
    }
    const float inv_n = 1.f / (4.f * (float)nf4);
    const float mean = warp_sum(sm) * inv_n;
    float q = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        if (lane + 32 * m < nf4) {
            v[m].x -= mean; v[m].y -= mean; v[m].z -= mean; v[m].w -= mean;
            q = fmaf(v[m].x, v[m].x, fmaf(v[m].y, v[m].y, fmaf(v[m].z, v[m].z, fmaf(v[m].w, v[m].w, q))));
        }
    }
    const float inv = rsqrtf(warp_sum(q) * inv_n + eps);   // every lane's loads are done
    if ((reinterpret_cast<uintptr_t>(row) & 127u) == 0)
        for (int li = lane; li < nf4 / 8; li += 32)           // 8 pieces per 128-byte line
            asm volatile("discard.global.L2 [%0], 128;" ::"l"(row + 32 * li) : "memory");
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        const int i = lane + 32 * m;
        if (i < nf4) {
            const float4 g = __ldg(reinterpret_cast<const float4*>(gamma) + i);
            const float4 bb = __ldg(reinterpret_cast<const float4*>(beta) + i);
            __nv_bfloat162 lo = __floats2bfloat162_rn(fmaf(v[m].x * inv, g.x, bb.x), fmaf(v[m].y * inv, g.y, bb.y));
            __nv_bfloat162 hi = __floats2bfloat162_rn(fmaf(v[m].z * inv, g.z, bb.z), fmaf(v[m].w * inv, g.w, bb.w));
            reinterpret_cast<uint2*>(orow)[i] =
                make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
        }
    }
}

// The LayerNorm workers of a fused launch: the extra CTAs (blockIdx.x >= units) and the CTA
// of every unit that is already complete (the fast kernel finished it), so that when the
// fast kernel did most of the work most of the device normalises.  A worker takes the next
// 64-token block (b, chunk c), in chunk-major order, from a counter after the progress
// words; warp 0 waits until every head's unit owning chunk c has published a progress past
// c (bounded; a unit that gave up publishes INT_MIN and the block is skipped), then each
// warp normalises rows.  Nothing waits for the workers, and the cooperative launch keeps
// them co-resident with the units they wait for.
__device__ void ln_blocks(Smem& s, const LnFuse& ln, const float* y_raw, int T, int H,
                          const Segments& seg, int units, int* status, long long budget) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nbh = units / seg.P, B = nbh / H, NCt = (T + C - 1) / C;
    const int nf4 = H * 16;
    const int blocks = B * NCt;
    for (;;) {
        if (warp == 0) {
            int rb = 0;
            if (lane == 0) rb = atomicAdd(ln.progress + units, 1);
            rb = __shfl_sync(0xffffffffu, rb, 0);
            bool ok = true;
            const int c = rb / B, b = rb - (rb / B) * B;
            const int p = min(c / seg.seg_chunks, seg.P - 1);
            for (int h = lane; rb < blocks && h < H; h += 32) {
                const int* w = ln.progress + (size_t)p * nbh + b * H + h;
                const long long t0 = clock64();
                int v = ld_acquire_gpu(w);
                while (v >= 0 && v <= c) {
                    if (clock64() - t0 > budget) {
                        v = -1;
                        break;
                    }
                    __nanosleep(500);
                    v = ld_acquire_gpu(w);
                }
                ok = ok && v > c;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (lane == 0) {
                s.ln_rb = rb;
                s.ln_go = ok ? 1 : 0;
            }
        }
        __syncthreads();
        const int rb = s.ln_rb;
        const bool go = s.ln_go != 0;
        __syncthreads();   // every warp has read the block before warp 0 takes the next one
        if (rb >= blocks) break;
        if (!go) {
            if (tid == 0) atomicExch(status, 1);
            continue;
        }
        const int c = rb / B, b = rb - (rb / B) * B;
        const int t_end = min(T, (c + 1) * C);
        for (int t = c * C + warp; t < t_end; t += kThreads / 32) {
            const size_t at = ((size_t)b * T + t) * (size_t)(H * 64);
            ln_row_warp(y_raw + at, ln.out + at, ln.gamma, ln.beta, ln.eps, nf4, lane);
        }
    }
}

// kC2: Finch-C2 exact form -- key k (1 - w), no static bonus, second value uprime added.
// kGN: base form with the GroupNorm + gate output stage (gn).
// kQ: no bonus, query r (1 - w) (Variant::query_c2).
template <bool kC2, bool kGN, bool kQ>
__global__ void __launch_bounds__(kThreads, 1)
wkv6_chunked_kernel(const __grid_constant__ CUtensorMap tm_r, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ u,
                    const float* s_in, float* s_out, float* __restrict__ y_raw,
                    const __nv_bfloat16* __restrict__ uprime, const GnOut gn, int T, int H, Segments seg, int* status, const int* start_chunk,
                    const float* handoff_state, long long spin_budget, long long drain_budget,
                    const LnFuse ln, int units) {
    extern __shared__ uint8_t smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if ((int)blockIdx.x >= units) {   // a LayerNorm CTA of a fused launch
        ln_blocks(s, ln, y_raw, T, H, seg, units, status, spin_budget);
        return;
    }
    // unit: segment pseg of sequence bh, absolute chunks c_begin .. NC - 1
    const int unit = blockIdx.x, nbh = units / seg.P;
    const int bh = unit % nbh, pseg = unit / nbh, b = bh / H, h = bh - (bh / H) * H;
    const int c_begin = pseg * seg.seg_chunks;
    const int NC = min((T + C - 1) / C, c_begin + seg.seg_chunks);
    // resume point: chunks before n0 (and the state entering n0) came from the fast kernel
    const int n0 = start_chunk ? start_chunk[unit] : c_begin;
    // LayerNorm fused: the rows before n0 (the fast kernel's, or another unit's) are stored
    if (ln.progress != nullptr && tid == 0)
        st_release_gpu(ln.progress + unit, (n0 < 0 || n0 >= NC) ? INT_MAX : n0);
    if (n0 < 0 || n0 >= NC) {             // this unit is already complete
        if (ln.progress != nullptr)       // its CTA normalises instead
            ln_blocks(s, ln, y_raw, T, H, seg, units, status, spin_budget);
        return;
    }
    const float* state0 = start_chunk ? handoff_state + (size_t)unit * 4096
                        : pseg > 0    ? seg.s_mid + ((size_t)bh * (seg.P - 1) + (pseg - 1)) * 4096
                        : s_in        ? s_in + (size_t)bh * 4096
                                      : nullptr;
    if (pseg < seg.P - 1) s_out = nullptr;   // only the last segment's final state is the output

    // ------------------------------------------------------------ set-up
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) ptx::mbar_init(&s.full[i], 1);
        ptx::mbar_init(&s.mma1u, 1);
        ptx::mbar_init(&s.mma1, 1);
        ptx::mbar_init(&s.mma2, 1);
        ptx::fence_mbar_init();
        s.abort = 0;
        ptx::prefetch_tensormap(&tm_r);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_w);
        ptx::prefetch_tensormap(&tm_y);
    }
    if (tid < 64) s.u[tid] = (kC2 || kQ) ? 0.f : u[h * 64 + tid];
    if (warp == 0) ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    // zero the operand tiles once, so that rows an MMA reads but never uses hold finite data
    for (int i = tid; i < (int)(sizeof(s.q) + sizeof(s.kk)) / 16; i += kThreads)
        reinterpret_cast<uint4*>(s.q)[i] = make_uint4(0, 0, 0, 0);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    auto issue_load = [&](int chunk) {
        const int st = (chunk - n0) % kStages;
        const int t0 = chunk * C;
        if (!gw_check(status, chunk >= n0 && chunk < NC && t0 < T && h < H && b < nbh / H)) return;
        ptx::mbar_arrive_expect_tx(&s.full[st], 4 * kTile);
        ptx::tma_load_4d(s.in[st][0], &tm_r, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][1], &tm_k, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][2], &tm_v, &s.full[st], 0, h, t0, b);
        ptx::tma_load_4d(s.in[st][3], &tm_w, &s.full[st], 0, h, t0, b);
    };
    if (tid == 0)
        for (int c = n0; c < n0 + kStages && c < NC; ++c) issue_load(c);

    // ------------------------------------------------------------ state in registers
    // warp w: TMEM sub-partition q = w % 4 (rows 16q .. 16q+15 in its lanes 0..15), columns
    // 32 hh .. 32 hh + 31.  The state and the output take a row on every lane: row
    // 16q + (l & 15), 16 columns from cb = 32 hh + 16 (l >> 4) (the two-half TMEM load).
    const int q = warp & 3, hh = warp >> 2;
    const int row = 16 * q + (lane & 15);          // state row i / token row t of this lane
    const int cb = 32 * hh + 16 * (lane >> 4);     // its first state / output column
    const int cc0 = cb >> 3;                       // its first 16-byte chunk of a tile row
    const uint32_t tlane = (uint32_t)(32 * q) << 16;
    float S[16];
    {
        const float* src = state0 ? state0 + row * 64 + cb : nullptr;
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
            st_shared_v4(s.s_hi, sw_chunk(row, cc0 + cc), hi);
            st_shared_v4(s.s_lo, sw_chunk(row, cc0 + cc), lo);
        }
    }

    bool failed = false;
    int n = n0;
    int issued1 = -1, issued2 = -1;   // last chunk whose MMA group 1 / 2 thread 0 issued
    for (; n < NC; ++n) {
        const int m = n - n0;             // position since the start: stage and phase parity
        const int st = m % kStages;
        const int t0 = n * C;
        const int valid = min(C, T - t0);
        uint8_t* r_tile = s.in[st][0];
        uint8_t* k_tile = s.in[st][1];
        uint8_t* v_tile = s.in[st][2];
        uint8_t* w_tile = s.in[st][3];
        uint8_t* y_tile = s.ystage[m & 1];
        if (tid == 0) ptx::bulk_wait_read<1>();    // the store that last used y_tile has read it

        if (!ptx::mbar_wait(&s.full[st], (uint32_t)((m / kStages) & 1), spin_budget)) s.abort = 1;

        // -------------------------------------------------------- prep
        {
            const int cg = warp;                      // channels 8cg .. 8cg+7
            const int ta = 2 * lane, tb = ta + 1;     // tokens of this lane
            float rv[2][8], kv[2][8], wv[2][8];
            {
                float om[2][8];
                unpack8(*reinterpret_cast<const uint4*>(r_tile + sw_chunk(ta, cg)), rv[0]);
                unpack8(*reinterpret_cast<const uint4*>(r_tile + sw_chunk(tb, cg)), rv[1]);
                unpack8(*reinterpret_cast<const uint4*>(k_tile + sw_chunk(ta, cg)), kv[0]);
                unpack8(*reinterpret_cast<const uint4*>(k_tile + sw_chunk(tb, cg)), kv[1]);
                unpack8(*reinterpret_cast<const uint4*>(w_tile + sw_chunk(ta, cg)), om[0]);
                unpack8(*reinterpret_cast<const uint4*>(w_tile + sw_chunk(tb, cg)), om[1]);
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        wv[p][c] = (ta + p < valid) ? __expf(-__expf(om[p][c])) : 1.f;
                if (kC2) {
                    // normalised key k (1 - w), 1 - w = -expm1(-exp(omega)); level 0 reads the
                    // k tile itself, so it is rewritten in place (bf16, as the other levels)
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            kv[p][c] *= (ta + p < valid) ? -expm1f(-__expf(om[p][c])) : 0.f;
                    st_shared_v4(k_tile, sw_chunk(ta, cg), pack8(kv[0]));
                    st_shared_v4(k_tile, sw_chunk(tb, cg), pack8(kv[1]));
                }
                if (kQ) {   // query r (1 - w); level 0 reads the r tile itself: rewritten in place
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            rv[p][c] *= (ta + p < valid) ? -expm1f(-__expf(om[p][c])) : 0.f;
                    st_shared_v4(r_tile, sw_chunk(ta, cg), pack8(rv[0]));
                    st_shared_v4(r_tile, sw_chunk(tb, cg), pack8(rv[1]));
                }
            }
            // bonus partials: sum over this lane's 8 channels of r u k
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) acc = fmaf(rv[p][c] * s.u[8 * cg + c], kv[p][c], acc);
                s.bonus_part[cg][ta + p] = acc;
            }
            // level 1: blocks of 2 tokens, both in this lane
            float E[2][8], F[2][8], BP[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                E[0][c] = 1.f;
                E[1][c] = wv[0][c];
                F[0][c] = wv[1][c];
                F[1][c] = 1.f;
                BP[c] = wv[0][c] * wv[1][c];
            }
            auto write_level = [&](uint8_t* qtile, uint8_t* ktile, bool upper) {
                // rows of t's upper half use Q^l = r * E, rows of the lower half K^l = k * F
                float f[8];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) f[c] = upper ? rv[p][c] * E[p][c] : kv[p][c] * F[p][c];
                    st_shared_v4(upper ? qtile : ktile, sw_chunk(ta + p, cg), pack8(f));
                }
            };
            write_level(s.q[0], s.kk[0], (lane & 1) != 0);
#pragma unroll
            for (int l = 2; l <= 6; ++l) {
                const int sh = 1 << (l - 2);
                const bool upper = (lane & sh) != 0;  // t in the upper 2^(l-1) half of its block
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float sib = __shfl_xor_sync(0xffffffffu, BP[c], sh);
                    const float mE = upper ? sib : 1.f;
                    const float mF = upper ? 1.f : sib;
                    E[0][c] *= mE;
                    E[1][c] *= mE;
                    F[0][c] *= mF;
                    F[1][c] *= mF;
                    BP[c] *= sib;
                }
                if (l <= 5) write_level(s.q[l - 1], s.kk[l - 1], (lane & (1 << (l - 1))) != 0);
            }
            // level 6 = the whole chunk: Rt = r * E6 (all rows), Kt^T = (k * F6)^T, gamma
            {
                float f[8];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) f[c] = rv[p][c] * E[p][c];
                    st_shared_v4(s.rt, sw_chunk(ta + p, cg), pack8(f));
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int i = 8 * cg + c;
                    const uint32_t off = (uint32_t)(i * 128 + ((((lane >> 2)) ^ (i & 7)) << 4) + (lane & 3) * 4);
                    *reinterpret_cast<uint32_t*>(s.ktT + off) = pack2(kv[0][c] * F[0][c], kv[1][c] * F[1][c]);
                }
                if (lane == 0)
#pragma unroll
                    for (int c = 0; c < 8; ++c) s.gamma[8 * cg + c] = BP[c];
            }
        }
        ptx::fence_proxy_async_smem();
        __syncthreads();
        if (s.abort) { failed = true; break; }

        // -------------------------------------------------------- MMA 1
        // U and Y first, with a commit of their own: the state chain needs only U, and may
        // rewrite S_hi / S_lo once Y has read them, while the level products still run
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t a_kt = ptx::smem_addr(s.ktT), b_v = ptx::smem_addr(v_tile);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_U, ptx::desc_kmajor(a_kt + 32 * kq),
                              ptx::desc_mnmajor(b_v + 2048 * kq), IDESC_KM, kq > 0);
            const uint32_t a_rt = ptx::smem_addr(s.rt);
            const uint32_t b_hi = ptx::smem_addr(s.s_hi), b_lo = ptx::smem_addr(s.s_lo);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(a_rt + 32 * kq),
                              ptx::desc_mnmajor(b_hi + 2048 * kq), IDESC_KM, kq > 0);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(a_rt + 32 * kq),
                              ptx::desc_mnmajor(b_lo + 2048 * kq), IDESC_KM, 1);
            ptx::mma_commit(&s.mma1u);
            const uint32_t a_r = ptx::smem_addr(r_tile), b_k = ptx::smem_addr(k_tile);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_L0, ptx::desc_kmajor(a_r + 32 * kq),
                              ptx::desc_kmajor(b_k + 32 * kq), IDESC_KK, kq > 0);
#pragma unroll
            for (int l = 1; l <= 5; ++l) {
                const uint32_t a = ptx::smem_addr(s.q[l - 1]), bb = ptx::smem_addr(s.kk[l - 1]);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    ptx::mma_bf16(tmem + 64 * l, ptx::desc_kmajor(a + 32 * kq),
                                  ptx::desc_kmajor(bb + 32 * kq), IDESC_KK, kq > 0);
            }
            ptx::mma_commit(&s.mma1);
            issued1 = n;
        }
        // LayerNorm fused: the previous chunk's fp32 rows (stored before that chunk's last
        // barrier) are published to the LayerNorm CTAs here, where every warp waits for the
        // products anyway, so the fence's wait is off the chunk's critical path (warp 1:
        // thread 0 issues the copies and products)
        if (ln.progress != nullptr && tid == 32 && n > n0) {
            __threadfence();
            st_release_gpu(ln.progress + unit, n);
        }
        if (!ptx::mbar_wait(&s.mma1u, (uint32_t)(m & 1), spin_budget)) s.abort = 1;
        ptx::tc_fence_after();

        // -------------------------------------------------------- state chain
        {
            uint32_t U[16];
            ptx::tmem_ld16x2(tmem + tlane + COL_U + 32 * hh, U);
            ptx::tmem_wait_ld();
            const float g = s.gamma[row];
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(g, S[j], __uint_as_float(U[j]));
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = S[8 * cc + e];
                uint4 hi, lo;
                split8(f, hi, lo);
                st_shared_v4(s.s_hi, sw_chunk(row, cc0 + cc), hi);
                st_shared_v4(s.s_lo, sw_chunk(row, cc0 + cc), lo);
            }
        }

        if (!ptx::mbar_wait(&s.mma1, (uint32_t)(m & 1), spin_budget)) s.abort = 1;
        ptx::tc_fence_after();

        // -------------------------------------------------------- assemble A
        {
            // lane: token row t, key blocks g = gw + 2 hf (8 columns each) for gw = 4 hh + gg;
            // the warp loads block gw, its half-warp hf = 1 receives block gw + 2.  The rows'
            // block pair (2q, 2q+1) lies after all of the warp's 4 blocks, before all of them,
            // or inside them (hh = q / 2): a warp-uniform choice of loads.
            const int t = row;
            const int p = t & 7;
            const bool upper8 = (lane & 15) >= 8;  // t in block 2q+1 (else 2q)
            const int hf = lane >> 4;
            float bonus = 0.f;
#pragma unroll
            for (int g = 0; g < 8; ++g) bonus += s.bonus_part[g][t];
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int gw = 4 * hh + gg;
                const int g = gw + 2 * hf;       // this lane's key block
                float a[8];
                if (4 * hh > 2 * q + 1) {        // every block after t's pair: no pairs
#pragma unroll
                    for (int c = 0; c < 8; ++c) a[c] = 0.f;
                } else if (4 * hh + 3 < 2 * q) {
                    // every block before t's pair: one level, the same for both halves (gw and
                    // gw + 2 differ in bit 1 only, below the highest bit where they leave 2q)
                    const int lvl = 3 + (31 - __clz((2 * q) ^ gw));
                    uint32_t v[8];
                    ptx::tmem_ld16x2_8(tmem + tlane + 64 * lvl + 8 * gw, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 8; ++c) a[c] = __uint_as_float(v[c]);
                } else {
                    // t's pair among the warp's blocks: levels 0-3 for the pair's own blocks
                    // and level 4 for a block before it (q odd: half-warp 0's blocks)
                    uint32_t v0[8], v1[8], v2[8], v3[8], v4[8];
                    ptx::tmem_ld16x2_8(tmem + tlane + 0 + 8 * gw, v0);
                    ptx::tmem_ld16x2_8(tmem + tlane + 64 + 8 * gw, v1);
                    ptx::tmem_ld16x2_8(tmem + tlane + 128 + 8 * gw, v2);
                    ptx::tmem_ld16x2_8(tmem + tlane + 192 + 8 * gw, v3);
                    ptx::tmem_ld16x2_8(tmem + tlane + 256 + 8 * gw, v4);
                    ptx::tmem_wait_ld();
                    if (g < 2 * q) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) a[c] = __uint_as_float(v4[c]);
                    } else if (g <= 2 * q + 1) {
                        const bool diag = (g == 2 * q) ? !upper8 : upper8;  // s in t's own 8-block
                        const bool below = (g == 2 * q) && upper8;           // whole block before t
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            float x = 0.f;
                            if (below) {
                                x = __uint_as_float(v3[c]);
                            } else if (diag) {
                                if (c == p) {
                                    x = bonus;
                                } else if (c < p) {
                                    const int lvl = 31 - __clz(p ^ c);
                                    x = __uint_as_float(lvl == 0 ? v0[c] : (lvl == 1 ? v1[c] : v2[c]));
                                }
                            }
                            a[c] = x;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) a[c] = 0.f;
                    }
                }
                uint4 hi, lo;
                split8(a, hi, lo);
                st_shared_v4(s.q[0], sw_chunk(t, g), hi);
                st_shared_v4(s.q[1], sw_chunk(t, g), lo);
            }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        __syncthreads();
        if (s.abort) { failed = true; break; }

        // -------------------------------------------------------- MMA 2: Y += A V
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t a_hi = ptx::smem_addr(s.q[0]), a_lo = ptx::smem_addr(s.q[1]);
            const uint32_t b_v = ptx::smem_addr(v_tile);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(a_hi + 32 * kq),
                              ptx::desc_mnmajor(b_v + 2048 * kq), IDESC_KM, 1);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                ptx::mma_bf16(tmem + COL_Y, ptx::desc_kmajor(a_lo + 32 * kq),
                              ptx::desc_mnmajor(b_v + 2048 * kq), IDESC_KM, 1);
            ptx::mma_commit(&s.mma2);
            issued2 = n;
        }
        if (!ptx::mbar_wait(&s.mma2, (uint32_t)(m & 1), spin_budget)) s.abort = 1;
        ptx::tc_fence_after();

        // -------------------------------------------------------- epilogue
        {
            uint32_t Y[16];
            ptx::tmem_ld16x2(tmem + tlane + COL_Y + 32 * hh, Y);
            ptx::tmem_wait_ld();
            if (kC2 && row < valid) {   // the second value u'_t joins the readout
                const __nv_bfloat16* up = uprime + (((size_t)b * T + t0 + row) * H + h) * 64 + cb;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4*>(up + 8 * cc), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) Y[8 * cc + e] = __float_as_uint(__uint_as_float(Y[8 * cc + e]) + f[e]);
                }
            }
            if (kGN) {
                // base Finch's output stage: GroupNorm of the (token, head) row over its 64
                // channels (this lane's 16, the other half-warp's 16 by a shuffle, then the
                // other 32 from the partner warp), the head's affine, times the gate
                float sm = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) sm += __uint_as_float(Y[j]);
                const float mean16 = sm * (1.f / 16.f);
                float q16 = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float d = __uint_as_float(Y[j]) - mean16;
                    q16 = fmaf(d, d, q16);
                }
                // merge two 16-value parts: (mean, M2) of the 32 columns, the same on both lanes
                const float om16 = __shfl_xor_sync(0xffffffffu, mean16, 16);
                const float oq16 = __shfl_xor_sync(0xffffffffu, q16, 16);
                const float d16 = om16 - mean16;
                const float2 mo = make_float2(0.5f * (mean16 + om16), q16 + oq16 + 8.f * d16 * d16);
                if (lane < 16) s.gn_mom[hh][row] = mo;
                __syncthreads();
                {
                    const float2 ot = s.gn_mom[hh ^ 1][row];
                    const float d = ot.x - mo.x;
                    const float mean = 0.5f * (mo.x + ot.x);
                    const float inv = rsqrtf((mo.y + ot.y + 16.f * d * d) * (1.f / 64.f) + gn.eps);
                    const int c0 = h * 64 + cb;
                    const __nv_bfloat16* gp = static_cast<const __nv_bfloat16*>(gn.gate);
                    const size_t gbase = (((size_t)b * T + t0 + row) * H + h) * 64 + cb;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        float gt[8];
                        if (gp != nullptr && row < valid) {
                            unpack8(__ldg(reinterpret_cast<const uint4*>(gp + gbase + 8 * cc)), gt);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) gt[e] = 1.f;
                        }
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 8 * cc + e;
                            f[e] = fmaf((__uint_as_float(Y[j]) - mean) * inv, __ldg(gn.gamma + c0 + j),
                                        __ldg(gn.beta + c0 + j)) * gt[e];
                        }
                        st_shared_v4(y_tile, sw_chunk(row, cc0 + cc), pack8(f));
                    }
                }
            } else if (y_raw != nullptr) {
                // fp32 rows for the LayerNorm pass: 64 contiguous bytes per lane
                if (row < valid) {
                    float* dst = y_raw + (((size_t)b * T + t0 + row) * H + h) * 64 + cb;
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(dst + j) =
                            make_float4(__uint_as_float(Y[j]), __uint_as_float(Y[j + 1]),
                                        __uint_as_float(Y[j + 2]), __uint_as_float(Y[j + 3]));
                }
            } else {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(Y[8 * cc + e]);
                    st_shared_v4(y_tile, sw_chunk(row, cc0 + cc), pack8(f));
                }
            }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        __syncthreads();
        if (s.abort) { failed = true; break; }
        if (tid == 0) {
            if (y_raw == nullptr && gw_check(status, t0 >= 0 && t0 < T && h < H && b < nbh / H)) {
                ptx::tma_store_4d(&tm_y, y_tile, 0, h, t0, b);
                ptx::bulk_commit();
            }
            // every thread is past its reads of this stage and the MMAs that read it are done
            if (n + kStages < NC) {
                ptx::fence_proxy_async_smem();
                issue_load(n + kStages);
            }
        }
    }

    // ------------------------------------------------------------ finish / drain
    if (failed) {
        if (tid == 0) {
            atomicExch(status, 1);
            if (ln.progress != nullptr) st_release_gpu(ln.progress + unit, INT_MIN);
            // copies still in flight: chunks n .. min(NC, n + kStages) - 1 may have been issued
            for (int c = n; c < NC && c < n + kStages; ++c)
                ptx::mbar_wait(&s.full[(c - n0) % kStages], (uint32_t)(((c - n0) / kStages) & 1),
                               drain_budget);
            if (issued1 == n) ptx::mbar_wait(&s.mma1, (uint32_t)((n - n0) & 1), drain_budget);
            if (issued2 == n) ptx::mbar_wait(&s.mma2, (uint32_t)((n - n0) & 1), drain_budget);
        }
    } else {
        if (s_out != nullptr) {
            float* dst = s_out + (size_t)bh * 4096 + row * 64 + cb;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (ln.progress != nullptr && tid == 32) {   // the last chunk's rows
            __threadfence();
            st_release_gpu(ln.progress + unit, INT_MAX);
        }
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

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
    static EncodeTiled fn = []() -> EncodeTiled {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiled>(p);
    }();
    return fn;
}

// [B][T][H][64] bf16 viewed as 4-D (D, H, T, B); box = 64 channels x 1 head x 64 tokens,
// 128-byte swizzle.  Rows past T read as zeros and are not written by stores.
bool make_token_map(CUtensorMap* m, const void* base, int B, int T, int H) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {64, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {64 * 2, (cuuint64_t)H * 64 * 2, (cuuint64_t)T * H * 64 * 2};
    const cuuint32_t box[4] = {64, 1, C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// [rows][cols] bf16, row stride `row_bytes` (a multiple of 16); box = 64 columns x
// box_rows rows, 128-byte swizzle.  Elements outside the matrix read as zeros.
bool make_matrix_map(CUtensorMap* m, const void* base, long rows, long cols, long row_bytes,
                     int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

size_t chunked_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_chunked_levels(const CUtensorMap* maps, const float* u, const float* s_in,
                                  float* s_out, float* y_raw, int B, int T, int H, Segments seg,
                                  Variant var, int* status, const int* start_chunk,
                                  const float* handoff_state, long long spin_budget,
                                  cudaStream_t st, const GnOut* gn, const LnFuse* ln,
                                  bool* ln_done) {
    if (ln_done) *ln_done = false;
    const size_t smem = chunked_smem_bytes();
    auto kernel = var.uprime     ? wkv6_chunked_kernel<true, false, false>
                  : gn           ? wkv6_chunked_kernel<false, true, false>
                  : var.query_c2 ? wkv6_chunked_kernel<false, false, true>
                                 : wkv6_chunked_kernel<false, false, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long drain = 4000000000LL;
    const int units = B * H * seg.P;
    const GnOut g = gn ? *gn : GnOut{nullptr, nullptr, 0.f, nullptr};
    // LayerNorm inside the launch: as many extra CTAs as stay co-resident with the units
    // (at most one per 64-token block), under a cooperative launch that guarantees it
    long ln_ctas = 0;
    if (ln != nullptr && y_raw != nullptr && gn == nullptr && H <= 32 && T > 0) {
        int dev = 0, nsm = 0, coop = 0, nb = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess &&
            coop != 0 &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kThreads, smem) == cudaSuccess) {
            ln_ctas = (long)nb * nsm - units;
            const long blocks = (long)B * ((T + C - 1) / C);
            if (ln_ctas > blocks) ln_ctas = blocks;
        } else {
            (void)cudaGetLastError();
        }
    }
    if (ln_ctas >= 1) {
        const LnFuse lf = *ln;
        void* args[] = {(void*)&maps[0], (void*)&maps[1], (void*)&maps[2], (void*)&maps[3],
                        (void*)&maps[4], (void*)&u, (void*)&s_in, (void*)&s_out, (void*)&y_raw,
                        (void*)&var.uprime, (void*)&g, (void*)&T, (void*)&H, (void*)&seg,
                        (void*)&status, (void*)&start_chunk, (void*)&handoff_state,
                        (void*)&spin_budget, (void*)&drain, (void*)&lf, (void*)&units};
        e = cudaLaunchCooperativeKernel((const void*)kernel, dim3((unsigned)(units + ln_ctas)),
                                        dim3(kThreads), args, smem, st);
        if (e != cudaErrorCooperativeLaunchTooLarge) {
            if (e == cudaSuccess && ln_done) *ln_done = true;
            return e;
        }
        // fewer slots than the occupancy query promised (another context holds SMs): the
        // refused launch queued nothing; run the units alone, the caller's pass normalises
        (void)cudaGetLastError();
    }
    const LnFuse none{nullptr, nullptr, nullptr, 0.f, nullptr};
    kernel<<<(unsigned)units, kThreads, smem, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], u, s_in, s_out, y_raw,
        static_cast<const __nv_bfloat16*>(var.uprime), g, T, H, seg, status, start_chunk,
        handoff_state, spin_budget, drain, none, units);
    return cudaGetLastError();
}

}  // namespace goldwkv
