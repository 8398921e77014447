// Backward pass of the WKV6 recurrence on CUDA cores, fp32 state and arithmetic.
//
// Forward (GoldFinch review page, section 3.4 "Recurrent state update and output", with the
// base-Finch bonus u): per (b,h)
//     y_t[j]  = sum_i r_t[i] S[i][j] + (sum_i r_t[i] u[i] k_t[i]) v_t[j]
//     S[i][j] = w_t[i] S[i][j] + k_t[i] v_t[j],     w_t = exp(-exp(omega_t)),
// S the state before token t.  Given dy and dS_T (the gradient of the final state), the
// chain rule gives, with G_t the gradient of the state after token t
// (G_{t-1} = diag(w_t) G_t + r_t^T dy_t, G_{T-1} = dS_T):
//     dr_t[i] = sum_j S_{t-1}[i][j] dy_t[j] + u[i] k_t[i] (v_t . dy_t)
//     dk_t[i] = sum_j G_t[i][j] v_t[j]      + u[i] r_t[i] (v_t . dy_t)
//     dv_t[j] = sum_i k_t[i] G_t[i][j]      + (sum_i r_t[i] u[i] k_t[i]) dy_t[j]
//     du[i]   = sum_{b,t} r_t[i] k_t[i] (v_t . dy_t),     dS_0 = G before the first token.
// The decay gradient is the sum of the pair terms (source token tau, reading token s) whose
// decay product contains w_t, i.e. tau < t < s.  Writing P_s = r_s * (dr_s without bonus)
// and Q_s = k_s * (dk_s without bonus) -- each the sum of the pair terms ending / starting at
// s -- and E = sum_j S_T[i][j] dS_T[i][j] for the pairs that end in the final state,
//     dlog w_t = E + sum_{s>t} P_s - sum_{s>=t} Q_s,     domega_t = dlog w_t * (-exp(omega_t)).
//
// Three sweeps, each a token-by-token scan like the forward recurrent kernel:
//   dr  rows of S (reduce over j), forward in time; also writes P, E and per-(b,h) du parts
//   dv  columns of G (reduce over i), reverse in time -- the forward recurrence with the
//       roles r <-> k, v -> dy run backwards
//   dk  rows of G, reverse in time, with the decay-gradient scan fused (needs P and E).
// The dr and dv sweeps run as one launch (blockIdx.z); the dk sweep follows; a small kernel
// sums du over the batch.  These scans are the whole fp32-I/O path.  With bf16 I/O they run
// only for a (b,h) that the tensor-core readouts (backward_tc_sm100.cu) hand back, and dv,
// exactly a forward recurrence in reversed time, runs through the chunked tensor-core
// prefill on time-reversed copies (reverse_tokens_kernel moves them).
//
// Work split: a CTA owns one (b,h) and 32 of the 64 rows (dr, dk) or columns (dv); each
// thread keeps a 4 x 4 block of the state in registers, and the sums over the other index
// finish over the 16 lanes of a half-warp by a reduce-scatter (reduce16x4).  Tokens are
// staged through shared memory in tiles of kTile (the next tile's 16-byte chunks held in
// registers meanwhile); per-token outputs are staged too and written coalesced per tile.
//
// Finch-C2's exact form (kC2): the key enters the state as kn_t = k_t (1 - w_t) and there
// is no bonus, so the dr and dv scans use kn in place of k (formed while staging), the dk
// scan yields dkn and returns dk = dkn (1 - w) with Q_t = kn_t dkn_t, and the decay gradient
// gains the direct term of kn on w: domega += dkn k w exp(omega).  du' = dy is the caller's
// copy.  With bf16 I/O dv goes through the chunked prefill here too, its query kn formed in
// the prefill's own staging; with fp32 I/O it is the dv scan with kn.
//
// Precision.  The identity subtracts, at every token, the pair terms that start at or after
// it; where w_t is tiny the result is tiny too and what is left is the rounding of those
// terms, times exp(omega_t).  With bf16 I/O that residue is far below the output rounding,
// and the row scans run in fp32.  With fp32 I/O (the precision path) the two row scans, P
// and E keep fp64, so the residue stays at fp64 rounding; the dv scan stays fp32.
#include "common.cuh"
#include "backward.h"

namespace goldwkv {

namespace {

constexpr int kHalf = 32;        // rows (or columns) per CTA
constexpr int kThreads = 128;    // 32 rows x 4 column quarters

// Accumulation type of the row scans and tokens per shared-memory tile, per I/O type.
template <typename IO> struct Prec {
    using Acc = float;
    static constexpr int kTile = 32;
};
template <> struct Prec<float> {
    using Acc = double;
    static constexpr int kTile = 16;
};

template <typename Acc, int kTile>
struct RowSmem {
    float b[kTile][kHeadSize];   // right factor of the update (v: dr sweep, dy: dk sweep)
    float q[kTile][kHeadSize];   // readout vector (dy: dr sweep, v: dk sweep)
    float a[kTile][kHalf];       // left factor of the update, this CTA's rows (k | r)
    float m[kTile][kHalf];       // the other of r / k, this CTA's rows (P or Q product)
    float w[kTile][kHalf];       // decay
    float ne[kTile][kHalf];      // -exp(omega): d w / d omega = w * ne  (dk sweep)
    Acc p[kTile][kHalf];         // P of the dr sweep (dk sweep)
    Acc o2[kTile][kHalf];        // staged P (dr sweep) / domega (dk sweep)
    float o1[kTile][kHalf];      // staged dr / dk
    float vdy[kTile];            // v_t . dy_t
    float u[kHalf];
};

template <int kTile>
struct ColSmem {
    float k[kTile][kHeadSize];
    float r[kTile][kHeadSize];
    float w[kTile][kHeadSize];
    float dy[kTile][kHalf];      // this CTA's columns
    float o[kTile][kHalf];       // staged dv
    float rku[kTile];            // sum_i r_t[i] u[i] k_t[i]
    float u[kHeadSize];
};

// Token-major element (b, t, h, c): ((b*T + t)*H + h)*64 + c.
__device__ __forceinline__ size_t tok_index(size_t xbase, int t, size_t tstride, int c) {
    return xbase + (size_t)t * tstride + c;
}

// Tiles move as 16-byte chunks: a thread loads its chunks of the NEXT tile into registers
// before computing the current one, and converts them into shared memory afterwards, so the
// global-memory latency hides behind a tile of work.  A tile of W channels x kTile tokens of
// type X has kTile * W * sizeof(X) / 16 chunks; chunk c covers elements
// [c * n, c * n + n) of the tile in token-major order, n = 16 / sizeof(X).  Every row of W
// channels is a whole number of chunks and starts 16-byte aligned in global memory.
template <typename X>
__device__ __forceinline__ uint4 load_chunk(const X* __restrict__ src, size_t xbase, size_t tstride,
                                            int t0, int nt, int colbase, int W, int c) {
    constexpr int n = 16 / sizeof(X);
    const int e = c * n, tt = e / W, col = e - (e / W) * W;
    if (tt >= nt) return make_uint4(0u, 0u, 0u, 0u);
    return __ldg(reinterpret_cast<const uint4*>(src + tok_index(xbase, t0 + tt, tstride,
                                                                  colbase + col)));
}

// The elements of a chunk as fp32 (bf16 / fp32 chunks) or as they are (fp64 chunks).
__device__ __forceinline__ void unpack(uint4 c, float (&f)[8]) {   // 8 bf16
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack(uint4 c, float (&f)[4]) {   // 4 fp32
    f[0] = __uint_as_float(c.x);
    f[1] = __uint_as_float(c.y);
    f[2] = __uint_as_float(c.z);
    f[3] = __uint_as_float(c.w);
}
__device__ __forceinline__ void unpack(uint4 c, double (&f)[2]) {  // 2 fp64
    f[0] = __hiloint2double((int)c.y, (int)c.x);
    f[1] = __hiloint2double((int)c.w, (int)c.z);
}

template <typename X> struct ChunkOf;
template <> struct ChunkOf<__nv_bfloat16> { using Elem = float; static constexpr int n = 8; };
template <> struct ChunkOf<float> { using Elem = float; static constexpr int n = 4; };
template <> struct ChunkOf<double> { using Elem = double; static constexpr int n = 2; };

// n fp32 values to dst (16-byte aligned) as 16-byte stores.
template <int n>
__device__ __forceinline__ void store_f32(float* dst, const float (&f)[n]) {
    static_assert(n % 4 == 0, "whole float4s");
#pragma unroll
    for (int j = 0; j < n; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
}

// Store chunk c of a token-major tile into dst (the tile flattened, same element order).
template <typename X>
__device__ __forceinline__ void put_chunk(uint4 raw, float* dst, int c) {
    float f[ChunkOf<X>::n];
    unpack(raw, f);
    store_f32(dst + c * ChunkOf<X>::n, f);
}
__device__ __forceinline__ void put_chunk_f64(uint4 raw, double* dst, int c) {
    *reinterpret_cast<uint4*>(dst + 2 * c) = raw;   // 2 fp64 values, bit for bit
}
__device__ __forceinline__ void put_chunk_acc(uint4 raw, float* dst, int c) {
    put_chunk<float>(raw, dst, c);
}
__device__ __forceinline__ void put_chunk_acc(uint4 raw, double* dst, int c) {
    put_chunk_f64(raw, dst, c);
}

// Sum of v over the 16 lanes of a half-warp for 4 rows at once (reduce-scatter): on return
// the lane holds the total of row 2*bit3 + bit2 of its lane index in v[0].
template <typename Acc>
__device__ __forceinline__ void reduce16x4(Acc (&v)[4], int lane) {
    const bool hi8 = lane & 8, hi4 = lane & 4;
    // lanes with bit 3 set keep rows 2, 3; the others rows 0, 1
    const Acc s0 = hi8 ? v[0] : v[2], s1 = hi8 ? v[1] : v[3];
    const Acc k0 = hi8 ? v[2] : v[0], k1 = hi8 ? v[3] : v[1];
    v[0] = k0 + __shfl_xor_sync(0xffffffffu, s0, 8);
    v[1] = k1 + __shfl_xor_sync(0xffffffffu, s1, 8);
    // bit 2 picks one of the two
    const Acc s2 = hi4 ? v[0] : v[1], k2 = hi4 ? v[1] : v[0];
    v[0] = k2 + __shfl_xor_sync(0xffffffffu, s2, 4);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// kRev == false: the dr sweep (a = k, m = r, b = v, q = dy, X0 = state_in), forward in time.
// kRev == true : the dk sweep (a = r, m = k, b = dy, q = v, X0 = dS_T), reverse in time, with
//                the decay-gradient scan (reads P and E written by the dr sweep).
// Thread (g, c) = (tid / 16, tid % 16) keeps the 4 x 4 block of rows 4g..4g+3 (of the CTA's
// 32) and columns 4c..4c+3: per token one 16-byte read each of the readout and update
// vectors (its 4 columns) and of the rows' a and w, the row sums finished over the 16 lanes
// of a half-warp by a reduce-scatter (5 shuffles for 4 rows).  Lane c % 4 == 0 of each
// group of four then owns row e = c / 4 (its outputs and running sums).
template <typename IO, bool kRev, bool kC2, typename Acc = typename Prec<IO>::Acc,
          int kTile = Prec<IO>::kTile>
__device__ __forceinline__ void row_sweep(RowSmem<Acc, kTile>& s, const IO* __restrict__ a_src,
                                          const IO* __restrict__ m_src,
                                          const IO* __restrict__ b_src,
                                          const IO* __restrict__ q_src,
                                          const IO* __restrict__ omega,
                                          const float* __restrict__ u, const float* x0,
                                          IO* __restrict__ out, Acc* __restrict__ P,
                                          IO* __restrict__ domega, Acc* __restrict__ E,
                                          const float* __restrict__ dS_T,
                                          float* __restrict__ du_part, float* x_final, int T,
                                          int H) {
    constexpr int D = kHeadSize;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - (bh / H) * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = tid >> 4, c = tid & 15;
    const int rowbase = blockIdx.y * kHalf;
    const int er = 2 * ((c >> 3) & 1) + ((c >> 2) & 1);   // row (of 4) this lane owns after
    const bool owner = (c & 3) == 0;                      // reduce16x4; one writer per row
    const int rl_own = 4 * g + er;                        // its local row 0..31

    if (tid < kHalf) s.u[tid] = kC2 ? 0.f : u[h * D + rowbase + tid];

    // X[e][f]: entry (rowbase + 4g + e, 4c + f)
    const size_t sbase = (size_t)bh * D * D + (size_t)(rowbase + 4 * g) * D + 4 * c;
    Acc X[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int f = 0; f < 4; ++f) X[e][f] = x0 ? (Acc)x0[sbase + (size_t)e * D + f] : Acc(0);

    const size_t tstride = (size_t)H * D;
    const size_t xbase = ((size_t)b * T * H + h) * D;
    const int ntile = (T + kTile - 1) / kTile;
    Acc du_acc = 0, accP = 0, accQ = 0;
    const Acc Ei = kRev ? E[(size_t)bh * D + rowbase + rl_own] : Acc(0);

    // chunk counts per thread: [kTile][64] and [kTile][32] tiles of IO, [kTile][32] of Acc
    constexpr int kFull = kTile * D * (int)sizeof(IO) / 16 / kThreads;
    constexpr int kRows = kTile * kHalf * (int)sizeof(IO) / 16 / kThreads;
    constexpr int kAcc = kTile * kHalf * (int)sizeof(Acc) / 16 / kThreads;
    static_assert(kFull * kThreads * 16 == kTile * D * (int)sizeof(IO) && kRows >= 1 &&
                      kRows * kThreads * 16 == kTile * kHalf * (int)sizeof(IO) &&
                      kAcc * kThreads * 16 == kTile * kHalf * (int)sizeof(Acc),
                  "tiles must split into whole chunks per thread");
    uint4 rb[kFull], rq[kFull], ra[kRows], rm[kRows], ro[kRows], rp[kAcc];
    auto fetch = [&](int it) {   // chunks of tile `it` (in sweep order) into registers
        const int t0 = (kRev ? ntile - 1 - it : it) * kTile, nt = min(kTile, T - t0);
#pragma unroll
        for (int k = 0; k < kFull; ++k) {
            rb[k] = load_chunk(b_src, xbase, tstride, t0, nt, 0, D, tid + k * kThreads);
            rq[k] = load_chunk(q_src, xbase, tstride, t0, nt, 0, D, tid + k * kThreads);
        }
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
            ra[k] = load_chunk(a_src, xbase, tstride, t0, nt, rowbase, kHalf, tid + k * kThreads);
            rm[k] = load_chunk(m_src, xbase, tstride, t0, nt, rowbase, kHalf, tid + k * kThreads);
            ro[k] = load_chunk(omega, xbase, tstride, t0, nt, rowbase, kHalf, tid + k * kThreads);
        }
        if (kRev) {
#pragma unroll
            for (int k = 0; k < kAcc; ++k)
                rp[k] = load_chunk(P, xbase, tstride, t0, nt, rowbase, kHalf, tid + k * kThreads);
        }
    };
    if (ntile > 0) fetch(0);

    for (int it = 0; it < ntile; ++it) {
        const int tile = kRev ? ntile - 1 - it : it;
        const int t0 = tile * kTile;
        const int nt = min(kTile, T - t0);
        __syncthreads();   // previous tile consumed and flushed
#pragma unroll
        for (int k = 0; k < kFull; ++k) {
            put_chunk<IO>(rb[k], &s.b[0][0], tid + k * kThreads);
            put_chunk<IO>(rq[k], &s.q[0][0], tid + k * kThreads);
        }
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
            constexpr int n = ChunkOf<IO>::n;
            put_chunk<IO>(rm[k], &s.m[0][0], tid + k * kThreads);
            float om[n], ne[n], w[n], av[n];
            unpack(ro[k], om);
            unpack(ra[k], av);
#pragma unroll
            for (int j = 0; j < n; ++j) {   // (padding tokens past T are never read)
                ne[j] = -expf(om[j]);
                w[j] = expf(ne[j]);
                if (kC2 && !kRev) av[j] *= -expm1f(ne[j]);   // the dr scan's kn = k (1 - w)
            }
            const int e0 = (tid + k * kThreads) * n;
            store_f32(&s.a[0][0] + e0, av);
            store_f32(&s.ne[0][0] + e0, ne);
            store_f32(&s.w[0][0] + e0, w);
        }
        if (kRev) {
#pragma unroll
            for (int k = 0; k < kAcc; ++k) put_chunk_acc(rp[k], &s.p[0][0], tid + k * kThreads);
        }
        __syncthreads();
        if (it + 1 < ntile) fetch(it + 1);   // in flight while this tile is computed
        for (int tt = warp * (kTile / 4); tt < (warp + 1) * (kTile / 4); ++tt) {
            const float p = warp_sum(s.b[tt][lane] * s.q[tt][lane] +
                                     s.b[tt][lane + 32] * s.q[tt][lane + 32]);
            if (lane == 0) s.vdy[tt] = p;
        }
        __syncthreads();

        for (int st = 0; st < nt; ++st) {
            const int tt = kRev ? nt - 1 - st : st;
            const float4 qv = *reinterpret_cast<const float4*>(&s.q[tt][4 * c]);
            const float4 bv = *reinterpret_cast<const float4*>(&s.b[tt][4 * c]);
            const float4 av = *reinterpret_cast<const float4*>(&s.a[tt][4 * g]);
            const float4 wv = *reinterpret_cast<const float4*>(&s.w[tt][4 * g]);
            const Acc qf[4] = {qv.x, qv.y, qv.z, qv.w}, bf[4] = {bv.x, bv.y, bv.z, bv.w};
            const Acc ae[4] = {av.x, av.y, av.z, av.w}, we[4] = {wv.x, wv.y, wv.z, wv.w};
            Acc part[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                Acc a0 = X[e][0] * qf[0], a1 = X[e][1] * qf[1];
                a0 += X[e][2] * qf[2];
                a1 += X[e][3] * qf[3];
                part[e] = a0 + a1;
#pragma unroll
                for (int f = 0; f < 4; ++f) X[e][f] = we[e] * X[e][f] + ae[e] * bf[f];
            }
            reduce16x4(part, lane);
            if (owner) {
                const Acc acc = part[0];
                const Acc vdy = s.vdy[tt], mi = s.m[tt][rl_own], ai = s.a[tt][rl_own];
                if (kC2 && kRev) {
                    // acc = dkn; m = k: kn = k (1 - w), dk = dkn (1 - w), and kn's own
                    // dependence on w adds -dkn k w to the gradient of w (before the chain
                    // factor d w / d omega = w ne)
                    const float ne = s.ne[tt][rl_own];
                    const Acc omw = (Acc)(-expm1f(ne)), wv = s.w[tt][rl_own];
                    s.o1[tt][rl_own] = (float)(acc * omw);
                    accQ += mi * omw * acc;               // Q_t with the source value kn_t
                    s.o2[tt][rl_own] = (Ei + accP - accQ - acc * mi * wv) * (Acc)ne;
                    accP += s.p[tt][rl_own];
                } else {
                    const Acc bonus = (Acc)s.u[rl_own] * ai * vdy;
                    s.o1[tt][rl_own] = (float)(acc + bonus);
                    if (!kRev) {
                        s.o2[tt][rl_own] = mi * acc;      // P_t: pair terms ending at t
                        du_acc += mi * ai * vdy;
                    } else {
                        accQ += mi * acc;                 // Q_t: pair terms starting at t
                        s.o2[tt][rl_own] = (Ei + accP - accQ) * (Acc)s.ne[tt][rl_own];
                        accP += s.p[tt][rl_own];
                    }
                }
            }
        }
        __syncthreads();
        for (int idx = tid; idx < nt * kHalf; idx += kThreads) {
            const int tt = idx / kHalf, cc = idx - (idx / kHalf) * kHalf;
            const size_t gi = tok_index(xbase, t0 + tt, tstride, rowbase + cc);
            out[gi] = from_f32<IO>(s.o1[tt][cc]);
            if (!kRev) P[gi] = s.o2[tt][cc];
            else domega[gi] = from_f32<IO>((float)s.o2[tt][cc]);
        }
    }

    if (!kRev) {
        Acc ev[4] = {0, 0, 0, 0};
        if (dS_T) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int f = 0; f < 4; ++f) ev[e] += X[e][f] * (Acc)dS_T[sbase + (size_t)e * D + f];
        }
        reduce16x4(ev, lane);
        if (owner) {
            E[(size_t)bh * D + rowbase + rl_own] = ev[0];
            du_part[(size_t)bh * D + rowbase + rl_own] = (float)du_acc;
        }
    } else if (x_final) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int f = 0; f < 4; ++f) x_final[sbase + (size_t)e * D + f] = (float)X[e][f];
    }
}

// The dv sweep: columns of G, reverse in time (the forward recurrence with r <-> k, v -> dy).
// Thread (g, c) = (tid / 16, tid % 16) keeps the 4 x 4 block of rows 4c..4c+3 and columns
// 4g..4g+3 (of the CTA's 32): per token one 16-byte read each of its rows' k, r and w and of
// its columns' dy; the column sums finish over the 16 lanes of a half-warp (reduce16x4),
// and lane c % 4 == 0 of each group of four owns column f = c / 4.
template <typename IO, bool kC2, int kTile = Prec<IO>::kTile>
__device__ __forceinline__ void col_sweep(ColSmem<kTile>& s, const IO* __restrict__ r,
                                          const IO* __restrict__ k, const IO* __restrict__ omega,
                                          const IO* __restrict__ dy, const float* __restrict__ u,
                                          const float* __restrict__ dS_T, IO* __restrict__ dv,
                                          int T, int H) {
    constexpr int D = kHeadSize;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - (bh / H) * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = tid >> 4, c = tid & 15;
    const int colbase = blockIdx.y * kHalf;
    const int fr = 2 * ((c >> 3) & 1) + ((c >> 2) & 1);   // column (of 4) this lane owns
    const bool owner = (c & 3) == 0;
    const int jl_own = 4 * g + fr;                        // its local column 0..31

    if (tid < D) s.u[tid] = kC2 ? 0.f : u[h * D + tid];

    // G[e][f]: entry (row 4c + e, column colbase + 4g + f)
    const size_t sbase = (size_t)bh * D * D + (size_t)(4 * c) * D + colbase + 4 * g;
    float G[4][4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int f = 0; f < 4; ++f) G[e][f] = dS_T ? dS_T[sbase + (size_t)e * D + f] : 0.f;

    const size_t tstride = (size_t)H * D;
    const size_t xbase = ((size_t)b * T * H + h) * D;
    const int ntile = (T + kTile - 1) / kTile;
    constexpr int kFull = kTile * D * (int)sizeof(IO) / 16 / kThreads;
    constexpr int kCols = kTile * kHalf * (int)sizeof(IO) / 16 / kThreads;
    static_assert(kFull * kThreads * 16 == kTile * D * (int)sizeof(IO) && kCols >= 1 &&
                      kCols * kThreads * 16 == kTile * kHalf * (int)sizeof(IO),
                  "tiles must split into whole chunks per thread");
    uint4 rr[kFull], rk[kFull], ro[kFull], rd[kCols];
    auto fetch = [&](int it) {   // chunks of tile `it` (reverse order) into registers
        const int t0 = (ntile - 1 - it) * kTile, nt = min(kTile, T - t0);
#pragma unroll
        for (int x = 0; x < kFull; ++x) {
            rr[x] = load_chunk(r, xbase, tstride, t0, nt, 0, D, tid + x * kThreads);
            rk[x] = load_chunk(k, xbase, tstride, t0, nt, 0, D, tid + x * kThreads);
            ro[x] = load_chunk(omega, xbase, tstride, t0, nt, 0, D, tid + x * kThreads);
        }
#pragma unroll
        for (int x = 0; x < kCols; ++x)
            rd[x] = load_chunk(dy, xbase, tstride, t0, nt, colbase, kHalf, tid + x * kThreads);
    };
    if (ntile > 0) fetch(0);
    for (int it = 0; it < ntile; ++it) {
        const int t0 = (ntile - 1 - it) * kTile;
        const int nt = min(kTile, T - t0);
        __syncthreads();
#pragma unroll
        for (int x = 0; x < kFull; ++x) {
            constexpr int n = ChunkOf<IO>::n;
            put_chunk<IO>(rr[x], &s.r[0][0], tid + x * kThreads);
            float om[n], w[n], kv[n];
            unpack(ro[x], om);
            unpack(rk[x], kv);
#pragma unroll
            for (int e = 0; e < n; ++e) {
                w[e] = decay_from_logit(om[e]);
                if (kC2) kv[e] *= -expm1f(-expf(om[e]));   // kn = k (1 - w)
            }
            store_f32(&s.w[0][0] + (tid + x * kThreads) * n, w);
            store_f32(&s.k[0][0] + (tid + x * kThreads) * n, kv);
        }
#pragma unroll
        for (int x = 0; x < kCols; ++x) put_chunk<IO>(rd[x], &s.dy[0][0], tid + x * kThreads);
        __syncthreads();
        if (it + 1 < ntile) fetch(it + 1);
        for (int tt = warp * (kTile / 4); tt < (warp + 1) * (kTile / 4); ++tt) {
            const float p = warp_sum(s.r[tt][lane] * s.u[lane] * s.k[tt][lane] +
                                     s.r[tt][lane + 32] * s.u[lane + 32] * s.k[tt][lane + 32]);
            if (lane == 0) s.rku[tt] = p;
        }
        __syncthreads();

        for (int st = 0; st < nt; ++st) {
            const int tt = nt - 1 - st;
            const float4 kv = *reinterpret_cast<const float4*>(&s.k[tt][4 * c]);
            const float4 rv = *reinterpret_cast<const float4*>(&s.r[tt][4 * c]);
            const float4 wv = *reinterpret_cast<const float4*>(&s.w[tt][4 * c]);
            const float4 dv4 = *reinterpret_cast<const float4*>(&s.dy[tt][4 * g]);
            const float ke[4] = {kv.x, kv.y, kv.z, kv.w}, re[4] = {rv.x, rv.y, rv.z, rv.w};
            const float we[4] = {wv.x, wv.y, wv.z, wv.w}, df[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
            float part[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                float a0 = ke[0] * G[0][f], a1 = ke[1] * G[1][f];
                a0 = fmaf(ke[2], G[2][f], a0);
                a1 = fmaf(ke[3], G[3][f], a1);
                part[f] = a0 + a1;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int f = 0; f < 4; ++f) G[e][f] = fmaf(we[e], G[e][f], re[e] * df[f]);
            reduce16x4(part, lane);
            if (owner) s.o[tt][jl_own] = fmaf(s.rku[tt], s.dy[tt][jl_own], part[0]);
        }
        __syncthreads();
        for (int idx = tid; idx < nt * kHalf; idx += kThreads) {
            const int tt = idx / kHalf, cc = idx - (idx / kHalf) * kHalf;
            dv[tok_index(xbase, t0 + tt, tstride, colbase + cc)] = from_f32<IO>(s.o[tt][cc]);
        }
    }
}

template <typename IO>
struct SweepSmem {
    using Row = RowSmem<typename Prec<IO>::Acc, Prec<IO>::kTile>;
    using Col = ColSmem<Prec<IO>::kTile>;
    static constexpr size_t kBytes = sizeof(Row) > sizeof(Col) ? sizeof(Row) : sizeof(Col);
};

// blockIdx.z == 0: dr sweep; blockIdx.z == 1: dv sweep.
template <typename IO, bool kC2>
__global__ void __launch_bounds__(kThreads, 4)   // 4 CTAs (16 warps) per SM
wkv6_bwd_dr_dv_kernel(const IO* __restrict__ r, const IO* __restrict__ k,
                      const IO* __restrict__ v, const IO* __restrict__ omega,
                      const float* __restrict__ u, const float* state_in, const IO* __restrict__ dy,
                      const float* __restrict__ dS_T, IO* __restrict__ dr, IO* __restrict__ dv,
                      typename Prec<IO>::Acc* __restrict__ P, typename Prec<IO>::Acc* __restrict__ E,
                      float* __restrict__ du_part, int T, int H, const int* dr_only) {
    using Sm = SweepSmem<IO>;
    __shared__ __align__(16) unsigned char smem[Sm::kBytes];
    if (blockIdx.z == 0 && dr_only != nullptr && dr_only[blockIdx.x] == 0) return;
    if (blockIdx.z == 0)
        row_sweep<IO, false, kC2>(*reinterpret_cast<typename Sm::Row*>(smem), k, r, v, dy, omega, u,
                             state_in, dr, P, nullptr, E, dS_T, du_part, nullptr, T, H);
    else
        col_sweep<IO, kC2>(*reinterpret_cast<typename Sm::Col*>(smem), r, k, omega, dy, u, dS_T, dv,
                      T, H);
}

template <typename IO, bool kC2>
__global__ void __launch_bounds__(kThreads, 4)   // 4 CTAs (16 warps) per SM
wkv6_bwd_dk_domega_kernel(const IO* __restrict__ r, const IO* __restrict__ k,
                          const IO* __restrict__ v, const IO* __restrict__ omega,
                          const float* __restrict__ u, const IO* __restrict__ dy,
                          const float* __restrict__ dS_T, IO* __restrict__ dk,
                          IO* __restrict__ domega, typename Prec<IO>::Acc* __restrict__ P,
                          typename Prec<IO>::Acc* __restrict__ E, float* dS_0, int T, int H,
                          const int* dk_only) {
    if (dk_only != nullptr && dk_only[blockIdx.x] == 0) return;
    __shared__ __align__(16) typename SweepSmem<IO>::Row s;
    row_sweep<IO, true, kC2>(s, r, k, dy, v, omega, u, dS_T, dk, P, domega, E, nullptr, nullptr, dS_0,
                        T, H);
}

// dst[i][b][t][h][:] = src[i][b][T-1-t][h][:] for n bf16 tensors [B][T][H][64]: 16-byte moves
struct ReverseArgs {
    const uint4* src[kMaxReverse];
    uint4* dst[kMaxReverse];
};

// A CTA moves kRows token rows (H*8 16-byte chunks each) of all kN tensors per step, every
// load of the step issued before its first store: kRows * kN = 8-10 loads in flight per
// thread, whatever the number of tensors (the destinations may not alias the sources, so
// nothing else would let a store wait behind the next load).
template <int kN>
__global__ void __launch_bounds__(256) reverse_tokens_kernel(ReverseArgs a, long rows, int T,
                                                             int row_chunks) {
    constexpr int kRows = kN >= 4 ? 2 : 8 / kN;
    for (long r0 = (long)blockIdx.x * kRows; r0 < rows; r0 += (long)gridDim.x * kRows) {
        for (int c = threadIdx.x; c < row_chunks; c += blockDim.x) {
            uint4 x[kRows][kN];
            long dst[kRows];
#pragma unroll
            for (int j = 0; j < kRows; ++j) {
                const long bt = r0 + j;
                dst[j] = -1;
                if (bt < rows) {
                    const long b = bt / T, t = bt - b * T;
                    const long src = (b * T + (T - 1 - t)) * row_chunks + c;
                    dst[j] = bt * row_chunks + c;
#pragma unroll
                    for (int i = 0; i < kN; ++i) x[j][i] = a.src[i][src];
                }
            }
#pragma unroll
            for (int j = 0; j < kRows; ++j)
                if (dst[j] >= 0) {
#pragma unroll
                    for (int i = 0; i < kN; ++i) a.dst[i][dst[j]] = x[j][i];
                }
        }
    }
}

// du[h][i] = sum_b du_part[b][h][i]  (fixed order: deterministic)
__global__ void wkv6_bwd_du_kernel(const float* __restrict__ du_part, float* __restrict__ du,
                                   int B, int H) {
    const int h = blockIdx.x, i = threadIdx.x;
    float acc = 0.f;
    for (int b = 0; b < B; ++b) acc += du_part[((size_t)b * H + h) * kHeadSize + i];
    du[(size_t)h * kHeadSize + i] = acc;
}

template <typename IO, bool kC2>
cudaError_t launch_typed(const void* r, const void* k, const void* v, const void* omega,
                         const float* u, const float* state_in, const void* dy,
                         const float* dstate_out, void* dr, void* dk, void* dv, void* domega,
                         float* du, float* dstate_in, void* P_, void* E_, float* du_part, int B,
                         int T, int H, bool with_dv, cudaStream_t st, const int* dr_only,
                         const int* dk_only, int phases) {
    using Acc = typename Prec<IO>::Acc;
    const IO *r_ = (const IO*)r, *k_ = (const IO*)k, *v_ = (const IO*)v, *o_ = (const IO*)omega,
             *dy_ = (const IO*)dy;
    Acc *P = static_cast<Acc*>(P_), *E = static_cast<Acc*>(E_);
    const unsigned bh = (unsigned)(B * H);
    cudaError_t e = cudaSuccess;
    if (phases & kPhaseDr) {
        wkv6_bwd_dr_dv_kernel<IO, kC2><<<dim3(bh, kHeadSize / kHalf, with_dv ? 2 : 1), kThreads, 0, st>>>(
            r_, k_, v_, o_, u, state_in, dy_, dstate_out, (IO*)dr, (IO*)dv, P, E, du_part, T, H,
            dr_only);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (phases & kPhaseDk) {
        wkv6_bwd_dk_domega_kernel<IO, kC2><<<dim3(bh, kHeadSize / kHalf), kThreads, 0, st>>>(
            r_, k_, v_, o_, u, dy_, dstate_out, (IO*)dk, (IO*)domega, P, E, dstate_in, T, H, dk_only);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (kC2 || !(phases & kPhaseDu)) return cudaSuccess;   // (no bonus u in Finch-C2's form)
    wkv6_bwd_du_kernel<<<H, kHeadSize, 0, st>>>(du_part, du, B, H);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const void* r, const void* k, const void* v, const void* omega,
                            const float* u, const float* state_in, const void* dy,
                            const float* dstate_out, void* dr, void* dk, void* dv, void* domega,
                            float* du, float* dstate_in, void* P, void* E, float* du_part,
                            int B, int T, int H, bool bf16, bool with_dv, bool c2,
                            cudaStream_t st, const int* dr_only, const int* dk_only, int phases) {
    using BF = __nv_bfloat16;
    if (c2)
        return bf16 ? launch_typed<BF, true>(r, k, v, omega, u, state_in, dy, dstate_out, dr, dk,
                                            dv, domega, du, dstate_in, P, E, du_part, B, T, H,
                                            with_dv, st, dr_only, dk_only, phases)
                    : launch_typed<float, true>(r, k, v, omega, u, state_in, dy, dstate_out, dr,
                                                dk, dv, domega, du, dstate_in, P, E, du_part, B,
                                                T, H, with_dv, st, dr_only, dk_only, phases);
    return bf16 ? launch_typed<BF, false>(r, k, v, omega, u, state_in, dy, dstate_out, dr, dk, dv,
                                          domega, du, dstate_in, P, E, du_part, B, T, H, with_dv,
                                          st, dr_only, dk_only, phases)
                : launch_typed<float, false>(r, k, v, omega, u, state_in, dy, dstate_out, dr, dk,
                                             dv, domega, du, dstate_in, P, E, du_part, B, T, H,
                                             with_dv, st, dr_only, dk_only, phases);
}

cudaError_t launch_reverse_tokens(const void* const* src, void* const* dst, int n, int B, int T,
                                  int H, cudaStream_t st) {
    if (n < 1 || n > kMaxReverse) return cudaErrorInvalidValue;
    if (B <= 0 || T <= 0 || H <= 0) return cudaSuccess;
    ReverseArgs a{};
    for (int i = 0; i < n; ++i) {
        a.src[i] = static_cast<const uint4*>(src[i]);
        a.dst[i] = static_cast<uint4*>(dst[i]);
    }
    const long rows = (long)B * T;
    const int row_chunks = H * 8;
    const int per_cta = n >= 4 ? 2 : 8 / n;
    const long need = (rows + per_cta - 1) / per_cta;
    const unsigned grid = (unsigned)(need < 148L * 32 ? need : 148L * 32);
    switch (n) {
        case 1: reverse_tokens_kernel<1><<<grid, 256, 0, st>>>(a, rows, T, row_chunks); break;
        case 2: reverse_tokens_kernel<2><<<grid, 256, 0, st>>>(a, rows, T, row_chunks); break;
        case 3: reverse_tokens_kernel<3><<<grid, 256, 0, st>>>(a, rows, T, row_chunks); break;
        case 4: reverse_tokens_kernel<4><<<grid, 256, 0, st>>>(a, rows, T, row_chunks); break;
        default: reverse_tokens_kernel<5><<<grid, 256, 0, st>>>(a, rows, T, row_chunks); break;
    }
    return cudaGetLastError();
}

}  // namespace goldwkv
