// Launcher of the WKV6 backward kernels (csrc/backward.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace goldwkv {

// Phases of launch_backward: the dr (and dv) sweep, the dk sweep with the decay gradient, the
// sum of du over the batch.
constexpr int kPhaseDr = 1, kPhaseDk = 2, kPhaseDu = 4, kPhaseAll = 7;

// Backward of the base recurrence: three token-by-token sweeps and a reduction of du over
// the batch.  Scratch the caller provides: P [B][T][H][64] and E [B*H][64] of the scans
// accumulation type (fp64 for fp32 I/O, fp32 for bf16 I/O), du_part [B*H][64] fp32.
// dstate_out / state_in may be null (zero); dstate_in may be null (not written).
// with_dv == false: dv is computed elsewhere (the caller's tensor-core path); dv unused.
// c2: Finch-C2's exact form (key k (1 - w), no bonus; u and du unused).
// dr_only != nullptr: the dr scan runs only for the (b,h) with dr_only[bh] != 0 (the others'
// dr, P, E and du_part were written by launch_bwd_dr_tc); dk_only likewise for the dk scan
// (dk, domega, dS_0 from launch_bwd_dk_tc and launch_bwd_domega).
cudaError_t launch_backward(const void* r, const void* k, const void* v, const void* omega,
                            const float* u, const float* state_in, const void* dy,
                            const float* dstate_out, void* dr, void* dk, void* dv, void* domega,
                            float* du, float* dstate_in, void* P, void* E, float* du_part,
                            int B, int T, int H, bool bf16, bool with_dv, bool c2,
                            cudaStream_t st, const int* dr_only = nullptr,
                            const int* dk_only = nullptr, int phases = kPhaseAll);

// dr of the base form (bf16 I/O) on the tensor cores (csrc/backward_tc_sm100.cu), one CTA per
// (b,h): writes dr and, as the CUDA-core dr scan does, P, E and du_part.  maps: dy, k, v,
// omega, dr ([B][T][H][64] bf16 token maps); r is read directly.  fallback[bh] = 1 for a
// (b,h) with a chunk whose decay range the one-sided factorisation cannot take (its outputs
// are then left to the scan), 0 otherwise.  status: set to 1 if a bounded wait expired.
// c2: Finch-C2's form (key k (1 - w), no bonus; u unused).
cudaError_t launch_bwd_dr_tc(const CUtensorMap* maps, const void* r, const float* u,
                             const float* state_in, const float* dS_T, float* P, float* E,
                             float* du_part, int* fallback, int B, int T, int H, int* status,
                             long long budget, cudaStream_t st, bool c2 = false);

// dk of the base form on the tensor cores, the same readout on time-reversed copies: maps
// v, r, dy, omega (all reversed) and any valid token map (unused); k in token order.  Writes
// dk and Q (the pair terms k_t (dk_t - bonus), fp32 [B][T][H][64]) in token order and dS_0
// (if non-null).  fallback / status as for launch_bwd_dr_tc.
// c2: Finch-C2's form: the readout is dkn, dk = dkn (1 - w), Q = k (1 - w) dkn, and D (fp32,
// token order) = dkn k w, the direct dependence of kn on w (D unused otherwise).
cudaError_t launch_bwd_dk_tc(const CUtensorMap* maps, const void* k, const float* u,
                             const float* dS_T, void* dk, float* Q, float* D, float* dS_0,
                             int* fallback, int B, int T, int H, int* status, long long budget,
                             cudaStream_t st, bool c2 = false);

// The column sums of X (P for half 0, Q for half 1; [B][T][H][64] fp32, token order) over
// each 64-token chunk into sums, B*H*ceil(T/64)*128 floats: sums[bh][n][64 * half + i].
cudaError_t launch_bwd_col_sums(const float* X, float* sums, int half, int B, int T, int H,
                                cudaStream_t st);

// domega (bf16) from P, Q (token order), their chunk sums (both halves) and E through the
// identity
//     dlog w_t = E + sum_{s>t} P_s - sum_{s>=t} Q_s - D_t,  domega_t = dlog w_t (-exp(omega_t));
// D: Finch-C2's direct term, or null (zero).
cudaError_t launch_bwd_domega(const float* P, const float* Q, const float* D, const float* sums,
                              const float* E, const void* omega, void* domega, int B, int T,
                              int H, cudaStream_t st);

constexpr int kMaxReverse = 5;

// dst[i] = src[i] with the token axis reversed, for n <= kMaxReverse bf16 tensors
// [B][T][H][64] (16-byte aligned, not overlapping).
cudaError_t launch_reverse_tokens(const void* const* src, void* const* dst, int n, int B, int T,
                                  int H, cudaStream_t st);

}  // namespace goldwkv
