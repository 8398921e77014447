// Kernel launchers behind the libgoldwkv C ABI (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>

#include "goldwkv.h"

namespace goldwkv {

// Which form of the time mixing: base Finch / RWKV-6 (static bonus u) when uprime is null;
// otherwise Finch-C2's exact form -- the key enters the state as k_t (1 - w_t), there is no
// static bonus, and the second value uprime (same layout and dtype as y) is added to the
// readout before LayerNorm.
struct Variant {
    const void* uprime;
    // query_c2 (base form, no bonus): the query is r (1 - w) instead of r -- Finch-C2's dv,
    // the forward recurrence in reversed time whose query is the normalised key k (1 - w)
    bool query_c2 = false;
};

// Token-by-token recurrence (fp32 math).  y_raw != nullptr: write fp32 un-normalised y
// there instead of y.
cudaError_t launch_recurrent(const void* r, const void* k, const void* v, const void* omega,
                             const float* u, const float* s_in, float* s_out, void* y,
                             float* y_raw, int B, int T, int H, bool bf16, Variant var,
                             cudaStream_t st);

// Output stage of a decode step: kind 0 none, 1 LayerNorm over each batch row's H*64
// outputs, 2 per-head GroupNorm times an optional gate (dtype io, layout of y).  LayerNorm:
// row_count [B] ints, zero before the call and left zero; y_raw [B][H][D] fp32 staging
// (null: y itself, fp32 I/O).
struct DecodeOut {
    int kind;
    const float* gamma;
    const float* beta;
    float eps;
    const void* gate;
    int* row_count;
    float* y_raw;
};

// One decode step, state in place, with its output stage fused.
cudaError_t launch_decode(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, float* state, void* y, const DecodeOut& out, int B,
                          int H, bool bf16, Variant var, cudaStream_t st);

// LayerNorm of `rows` rows of C fp32 values into `out` (fp32 or bf16); out may equal x.
cudaError_t launch_layernorm_rows(const float* x, const float* gamma, const float* beta,
                                  float eps, void* out, long rows, int C, bool bf16,
                                  cudaStream_t st);

// Per-head GroupNorm (rows of 64 = one head of one token; gamma/beta [H*64], head = row % H)
// then times gate (same layout as out, or null).  out may equal x (fp32).
cudaError_t launch_groupnorm_gate(const float* x, const float* gamma, const float* beta, float eps,
                                  const void* gate, void* out, long rows, int H, bool bf16,
                                  cudaStream_t st);

// ---- chunked tensor-core prefill (bf16 I/O)
// TMA descriptor of a [B][T][H][64] bf16 tensor: box 64 channels x 1 head x 64 tokens.
bool make_token_map(CUtensorMap* m, const void* base, int B, int T, int H);
// TMA descriptor of a [rows][cols] bf16 matrix, row stride row_bytes: box 64 columns x
// box_rows rows, 128-byte swizzle, zeros outside the matrix.
bool make_matrix_map(CUtensorMap* m, const void* base, long rows, long cols, long row_bytes,
                     int box_rows);

// Sequence split.  Every (b,h) sequence is cut into P segments of seg_chunks 64-token
// chunks (the last one may be shorter); the kernels below run one CTA per unit
// u = p * (B*H) + bh.  The state entering segment p > 0 is s_mid[bh][p-1] ([D][D] fp32),
// computed beforehand by launch_segment_states + launch_segment_carry.  P = 1: no split.
struct Segments {
    int P;
    int seg_chunks;
    const float* s_mid;
};

// State of each segment p < P-1 from a zero initial state, s_loc[bh][p] ([D][D]), and its
// log2 decay sum[bh][p][i] = log2 prod_{t in segment} w_t[i]; chunked on tcgen05 with the
// suffix factorisation (factors <= 1: no overflow for any decay).  maps: r, k, v, omega.
cudaError_t launch_segment_states(const CUtensorMap* maps, float* s_loc, float* log2g, int B,
                                  int T, int H, Segments seg, Variant var, int* status,
                                  long long budget, cudaStream_t st);
// s_mid[bh][p] = 2^log2g[bh][p] (rows) * s_in(p) + s_loc[bh][p], p = 0 .. P-2, in order, where
// s_in(0) = state_in (zero if null) and s_in(p) = s_mid[bh][p-1]; s_mid may alias s_loc.
cudaError_t launch_segment_carry(const float* state_in, const float* s_loc, const float* log2g,
                                 float* s_mid, int B, int H, int P, cudaStream_t st);
// The same chain over P segments laid out segment-major (s_loc [P][B*H][D][D], log2g
// [P][B*H][D]): s_in [P + 1][B*H][D][D], s_in[0] = state0 (zero if null), s_in[p + 1] =
// 2^log2g[p] (rows) * s_in[p] + s_loc[p].
cudaError_t launch_segment_carry_ranks(const float* state0, const float* s_loc,
                                       const float* log2g, float* s_in, int B, int H, int P,
                                       cudaStream_t st);

// Base Finch's output stage fused into the chunked kernels: per (token, head) GroupNorm over
// the head's 64 channels (biased variance, eps inside the square root), the per-channel
// affine gamma / beta ([H*64] fp32), then times gate (bf16, layout of y; null: no gate).
struct GnOut {
    const float* gamma;
    const float* beta;
    float eps;
    const void* gate;
};

// Fast path (one-sided decay factorisation, warp-specialised pipeline).  maps: r, k, v,
// omega.  For each unit it writes y (and, in the last segment, the final state), or stops at
// the first chunk whose decay range it cannot take and records that chunk (absolute index)
// in handoff_chunk[u] (-1: done) with the state entering it in handoff_state[u].
// y_raw != nullptr: fp32 y rows there instead of y.  gn != nullptr: y = GroupNorm + gate of
// the rows (base form only; y_raw must then be null).
cudaError_t launch_chunked_fast(const CUtensorMap* maps, const float* u, const float* s_in,
                                float* s_out, void* y, float* y_raw, int B, int T, int H,
                                Segments seg, Variant var, int* status, int* handoff_chunk,
                                float* handoff_state, long long budget, cudaStream_t st,
                                const GnOut* gn = nullptr);

// LayerNorm of the fp32 rows y_raw (a token's H heads) inside the level kernel's launch:
// extra CTAs, co-resident with the recurrence's (a cooperative launch), normalise the
// 64-token blocks of a batch row as soon as every head has published them (so do the CTAs
// of units the fast kernel already finished).  progress: one word per (b,h,segment) unit
// and a block counter after them, all zero before the launch; a unit stores, with release
// semantics, the absolute index of the first chunk whose rows it has not yet stored
// (INT_MAX: all; INT_MIN: it gave up).
struct LnFuse {
    int* progress;
    const float* gamma;
    const float* beta;
    float eps;
    __nv_bfloat16* out;   // y [B][T][H][64]
};

// Level-factorised path (any decay).  start_chunk == nullptr: every unit from its first
// chunk with its incoming state; otherwise unit u resumes at chunk start_chunk[u] (skipped if
// < 0) from handoff_state[u].  status: device word set to 1 if a bounded wait expired.
// gn: as for the fast path.  ln (y_raw != nullptr, H <= 32): LayerNorm into ln->out within
// the launch if the recurrence's CTAs leave room for at least one more co-resident CTA;
// *ln_done says whether it did (else the caller runs the LayerNorm pass).
cudaError_t launch_chunked_levels(const CUtensorMap* maps, const float* u, const float* s_in,
                                  float* s_out, float* y_raw, int B, int T, int H, Segments seg,
                                  Variant var, int* status, const int* start_chunk,
                                  const float* handoff_state, long long spin_budget,
                                  cudaStream_t st, const GnOut* gn = nullptr,
                                  const LnFuse* ln = nullptr, bool* ln_done = nullptr);
size_t chunked_smem_bytes();
size_t fast_smem_bytes();
size_t segment_smem_bytes();

// ---- prefill within a fixed workspace (the allocation-free entry point uses these)
// Bytes wkv6_prefill (WKV_ALGO_AUTO) needs when its sequence split is capped so that the
// workspace stays within `cap`: the split choose_segments makes if it fits, else the largest
// smaller one that does, else none (the result may then still exceed cap).  0 = no workspace.
size_t prefill_bytes_within(int B, int T, int H, int D, wkv_dtype io, bool with_ln, size_t cap);
// wkv6_prefill (WKV_ALGO_AUTO) with the split capped by workspace_bytes as above; same
// arguments, checks and results.  WKV_ERR_WORKSPACE when even the unsplit path does not fit.
wkv_status prefill_within(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, const float* state_in, float* state_out, void* y,
                          int B, int T, int H, int D, wkv_dtype io, const wkv_ln* ln,
                          void* workspace, size_t workspace_bytes, void* stream);

// The calling thread's current CUDA context, or null (none yet, or the driver entry point
// could not be had).  Makes no context current and does not synchronise.
CUcontext current_context();

}  // namespace goldwkv
