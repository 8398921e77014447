// GOLD's two matrix products on the tcgen05 tensor cores (GoldFinch review page, section 3.4
// "GOLD Key Compression and TokenCat Decompression"):
//     c_t   = x_t W_KD                                   compression, D -> Dc
//     k^D_t = RMSNorm(concat(x0_t, c_t) W_KU)            decompression, D + Dc -> D
//
// One kernel computes C [M][Nout] = [A1 | A2] [M][K1 + K2] . B^T with B [Nout][K1 + K2] (the
// weights are given as the rows of each map), bf16 operands, fp32 accumulation in TMEM.
// The concatenation is never formed: the k-blocks of A1 (x0) and then those of A2 (c) are
// loaded from their own tensors, each paired with the matching columns of B through a
// tensor map of its own, so K1 need not be a multiple of the k-block (elements outside a
// matrix load as zeros and add nothing).
//
// A CTA computes one 128-row x BN-column tile: warp 0 issues the TMA copies into a 4-stage
// ring, warp 1 issues the tcgen05 products and owns the TMEM accumulator, warps 2-5 read it
// back (one TMEM lane quarter each: thread = one output row) and store it, as bf16 or
// fp32, or -- for the decompression -- normalise it first: the CTAs holding one row block's
// column tiles form a thread-block cluster, each adds up its share of the row's sum of
// squares, the partial sums are exchanged through distributed shared memory, and every CTA
// scales its own columns.  The fp32 product never leaves the chip.
//
// Every mbarrier wait is bounded; on expiry the CTA records it in *status and skips the
// rest of its work, but still takes both cluster barriers so that no CTA of its cluster is
// left waiting.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "gold.h"
#include "internal.h"
#include "chunk_tiles.cuh"
#include "sm100_ptx.cuh"

namespace goldwkv {

namespace {

using tiles::ld_volatile;
using tiles::pack2;

constexpr int BM = 128, BK = 64;
// stages of the copy ring: sized so that two CTAs share an SM (one's epilogue overlaps the
// other's products)
template <int BN>
struct Stages {
    static constexpr int value = BN >= 256 ? 2 : 3;
};
constexpr int kThreads = 192;     // warp 0 copies, warp 1 products, warps 2-5 epilogue
constexpr int kEpiWarp0 = 2;
// waits for work already in flight (copies, products) before the CTA may exit: long, but
// bounded like every other wait
constexpr long long kDrainBudget = 4000000000LL;

enum Epi { kStoreBf16 = 0, kStoreF32 = 1, kRmsNorm = 2 };

template <int BN>
struct __align__(1024) GemmSmem {
    static constexpr int kStages = Stages<BN>::value;
    uint8_t a[kStages][BM * BK * 2];   // A tiles: 128 rows x 64 bf16 (128 B), 128B swizzle
    uint8_t b[kStages][BN * BK * 2];   // B tiles: BN rows x 64 bf16
    uint64_t full[kStages], empty[kStages], acc_full;
    float rowsum[BM];                  // RMSNorm: this CTA's partial sum of squares per row
    uint32_t tmem_base;
    int abort;
};

template <int BN>
struct Idesc {
    static constexpr uint32_t value = ptx::idesc_bf16(BM, BN, 0, 0);
};

// Bounded wait that records an expiry; false if this CTA has given up.
template <class Sm>
__device__ __forceinline__ bool wait_or_abort(Sm& s, uint64_t* bar, uint32_t parity,
                                              long long budget, int* status) {
    if (ld_volatile(&s.abort)) return false;
    if (ptx::mbar_wait(bar, parity, budget)) return true;
    s.abort = 1;
    atomicExch(status, 1);
    return false;
}

// 32 consecutive output values of one row, fp32, stored as bf16 or fp32 from column col0;
// ncols (a multiple of 8) bounds the columns
template <bool kF32>
__device__ __forceinline__ void store_row32(void* C, long ldc, long row, int col0, int ncols,
                                            const float (&v)[32]) {
    if (kF32) {
        float* p = static_cast<float*>(C) + row * ldc + col0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (col0 + 4 * q + 4 <= ncols)
                *reinterpret_cast<float4*>(p + 4 * q) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
        __nv_bfloat16* p = static_cast<__nv_bfloat16*>(C) + row * ldc + col0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (col0 + 8 * q + 8 <= ncols) {
                uint4 w;
                w.x = pack2(v[8 * q], v[8 * q + 1]);
                w.y = pack2(v[8 * q + 2], v[8 * q + 3]);
                w.z = pack2(v[8 * q + 4], v[8 * q + 5]);
                w.w = pack2(v[8 * q + 6], v[8 * q + 7]);
                *reinterpret_cast<uint4*>(p + 8 * q) = w;
            }
    }
}

template <int BN, int kEpi>
__global__ void __launch_bounds__(kThreads, 2)
gold_gemm_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                 const __grid_constant__ CUtensorMap tm_b1, const __grid_constant__ CUtensorMap tm_b2,
                 int nk1, int nk2, void* C, long ldc, long M, int ncols,
                 const float* __restrict__ gamma, float eps, int* status, long long budget) {
    using Sm = GemmSmem<BN>;
    constexpr int kStages = Sm::kStages;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tile = blockIdx.x, m_tile = blockIdx.y;
    const int nk = nk1 + nk2;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&s.full[i], 1);
            ptx::mbar_init(&s.empty[i], 1);
        }
        ptx::mbar_init(&s.acc_full, 1);
        ptx::fence_mbar_init();
        s.abort = 0;
        ptx::prefetch_tensormap(&tm_a1);
        ptx::prefetch_tensormap(&tm_b1);
        if (nk2 > 0) {
            ptx::prefetch_tensormap(&tm_a2);
            ptx::prefetch_tensormap(&tm_b2);
        }
    }
    if (warp == 1) ptx::tmem_alloc(&s.tmem_base, BN);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // ---- copies: k-block kb of A and B into stage kb % kStages
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int st = kb % kStages;
                if (kb >= kStages &&
                    !wait_or_abort(s, &s.empty[st], (uint32_t)((kb / kStages - 1) & 1), budget, status))
                    break;
                ptx::mbar_arrive_expect_tx(&s.full[st], (BM + BN) * BK * 2);
                const bool first = kb < nk1;
                const int kx = (first ? kb : kb - nk1) * BK;
                ptx::tma_load_2d(s.a[st], first ? &tm_a1 : &tm_a2, &s.full[st], kx, m_tile * BM);
                ptx::tma_load_2d(s.b[st], first ? &tm_b1 : &tm_b2, &s.full[st], kx, n_tile * BN);
                issued = kb + 1;
            }
            // every issued copy lands before the CTA may exit
            for (int kb = issued - kStages < 0 ? 0 : issued - kStages; kb < issued; ++kb)
                ptx::mbar_wait(&s.full[kb % kStages], (uint32_t)((kb / kStages) & 1), kDrainBudget);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- products: 4 x (M128 x BN x K16) per k-block, accumulated in TMEM
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int st = kb % kStages;
                ok = wait_or_abort(s, &s.full[st], (uint32_t)((kb / kStages) & 1), budget, status);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t a = ptx::smem_addr(s.a[st]), b = ptx::smem_addr(s.b[st]);
#pragma unroll
                for (int kq = 0; kq < BK / 16; ++kq)
                    ptx::mma_bf16(tmem, ptx::desc_kmajor(a + 32 * kq), ptx::desc_kmajor(b + 32 * kq),
                                  Idesc<BN>::value, (kb | kq) != 0);
                ptx::mma_commit(&s.empty[st]);   // stage st may be refilled once these are done
            }
            // the accumulator is complete (or, after an expiry, nothing more is in flight)
            ptx::mma_commit(&s.acc_full);
            ptx::mbar_wait(&s.acc_full, 0, kDrainBudget);
        }
    } else {
        // ---- epilogue: thread = one row of the tile (TMEM lane quarter warp % 4)
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const long grow = (long)m_tile * BM + row;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        bool ok = wait_or_abort(s, &s.acc_full, 0, budget, status);
        ptx::tc_fence_after();
        if (kEpi != kRmsNorm) {
            if (ok) {
#pragma unroll 1
                for (int cc = 0; cc < BN / 32; ++cc) {
                    uint32_t raw[32];
                    ptx::tmem_ld32(tmem + lane_base + 32 * cc, raw);
                    ptx::tmem_wait_ld();
                    const int col0 = n_tile * BN + 32 * cc;
                    if (grow < M && col0 < ncols) {
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
                        store_row32<kEpi == kStoreF32>(C, ldc, grow, col0, ncols, v);
                    }
                }
            }
        } else {
            // sum of squares of this CTA's columns of the row (columns past ncols are zeros)
            float ss = 0.f;
            if (ok) {
#pragma unroll 1
                for (int cc = 0; cc < BN / 32; ++cc) {
                    uint32_t raw[32];
                    ptx::tmem_ld32(tmem + lane_base + 32 * cc, raw);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float z = __uint_as_float(raw[i]);
                        ss = fmaf(z, z, ss);
                    }
                }
            }
            s.rowsum[row] = ss;
        }
        ptx::tc_fence_before();
    }

    __syncwarp();   // each warp converged again (lane 0 of warps 0 and 1 ran alone)
    if (kEpi == kRmsNorm) {
        // the row block's column tiles are this cluster's CTAs: exchange the partial sums
        ptx::cluster_sync();
        if (warp >= kEpiWarp0 && !ld_volatile(&s.abort)) {
            const int q = warp & 3;
            const int row = 32 * q + lane;
            const long grow = (long)m_tile * BM + row;
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            const uint32_t nrank = ptx::cluster_nctarank();
            float total = 0.f;
            for (uint32_t r = 0; r < nrank; ++r) total += ptx::ld_dsmem_f32(&s.rowsum[row], r);
            const float scale = rsqrtf(total / (float)ncols + eps);
            ptx::tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t raw[32];
                ptx::tmem_ld32(tmem + lane_base + 32 * cc, raw);
                ptx::tmem_wait_ld();
                const int col0 = n_tile * BN + 32 * cc;
                if (grow < M && col0 < ncols) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int col = min(col0 + i, ncols - 1);
                        v[i] = __uint_as_float(raw[i]) * scale * (gamma ? gamma[col] : 1.f);
                    }
                    store_row32<false>(C, ldc, grow, col0, ncols, v);
                }
            }
            ptx::tc_fence_before();
        }
        // no CTA leaves while another may still read its partial sums
        __syncwarp();
        ptx::cluster_sync();
    }

    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, BN);
    }
}

template <int BN, int kEpi>
size_t gemm_smem() {
    return sizeof(GemmSmem<BN>) + 1024;
}

template <int BN, int kEpi>
cudaError_t launch_gemm(const CUtensorMap* maps, int nk1, int nk2, void* C, long ldc, long M,
                        int ncols, const float* gamma, float eps, int* status, long long budget,
                        cudaStream_t st) {
    auto kernel = gold_gemm_kernel<BN, kEpi>;
    const size_t smem = gemm_smem<BN, kEpi>();
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned gx = (unsigned)((ncols + BN - 1) / BN);
    const unsigned gy = (unsigned)((M + BM - 1) / BM);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, gy, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (kEpi == kRmsNorm) {   // one cluster per row block: all its column tiles
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = gx;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    e = cudaLaunchKernelEx(&cfg, kernel, maps[0], maps[1], maps[2], maps[3], nk1, nk2, C, ldc, M,
                           ncols, gamma, eps, status, budget);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Tensor maps of [A1 | A2] and the matching column blocks of B ([Nout][K1 + K2]); A2 / B2
// are copies of A1 / B1 when K2 == 0 (never loaded).
bool make_maps(CUtensorMap* maps, const void* a1, long K1, const void* a2, long K2,
               const void* b, long nout, long M, int bn) {
    const long kb = (K1 + K2) * 2;
    if (!make_matrix_map(&maps[0], a1, M, K1, K1 * 2, BM)) return false;
    if (!make_matrix_map(&maps[2], b, nout, K1, kb, bn)) return false;
    if (K2 > 0) {
        if (!make_matrix_map(&maps[1], a2, M, K2, K2 * 2, BM)) return false;
        if (!make_matrix_map(&maps[3], static_cast<const __nv_bfloat16*>(b) + K1, nout, K2, kb, bn))
            return false;
    } else {
        maps[1] = maps[0];
        maps[3] = maps[2];
    }
    return true;
}

}  // namespace

bool gold_rmsnorm_fusable(int D) { return D <= 8 * 256; }

cudaError_t gold_gemm(const void* a1, long K1, const void* a2, long K2, const void* w, long nout,
                      long M, GoldOut out, void* C, const float* gamma, float eps, int* status,
                      long long budget, cudaStream_t st) {
    CUtensorMap maps[4];
    const int nk1 = (int)((K1 + BK - 1) / BK), nk2 = (int)((K2 + BK - 1) / BK);
    const bool narrow = nout <= 128;   // the compression's Dc: one 128-wide column tile
    if (!make_maps(maps, a1, K1, a2, K2, w, nout, M, narrow ? 128 : 256))
        return cudaErrorInvalidValue;
    const int nc = (int)nout;
    if (out == GoldOut::kRmsNormBf16) {
        if (narrow)
            return launch_gemm<128, kRmsNorm>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status,
                                              budget, st);
        return launch_gemm<256, kRmsNorm>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status,
                                          budget, st);
    }
    if (out == GoldOut::kF32) {
        if (narrow)
            return launch_gemm<128, kStoreF32>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status,
                                               budget, st);
        return launch_gemm<256, kStoreF32>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status,
                                           budget, st);
    }
    if (narrow)
        return launch_gemm<128, kStoreBf16>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status,
                                            budget, st);
    return launch_gemm<256, kStoreBf16>(maps, nk1, nk2, C, nout, M, nc, gamma, eps, status, budget,
                                        st);
}

}  // namespace goldwkv
