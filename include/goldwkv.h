/*
 * libgoldwkv -- the Finch-C2 / RWKV-6 time-mix WKV recurrence on NVIDIA B200 (sm_100a).
 *
 * What is computed (GoldFinch review page, section 3.4 "Finch-C2 Time Mixing"): per batch
 * row b and head h, with head size D = 64, a D x D fp32 state S whose rows i are key /
 * decay channels and whose columns j are value channels.  For each token t:
 *
 *     w_t[i]  = exp(-exp(omega_t[i]))                    ("Data-dependent decay")
 *     y_t[j]  = sum_i r_t[i] * S[i][j]
 *             + (sum_i r_t[i] * u[i] * k_t[i]) * v_t[j]   (base-Finch static bonus u)
 *     S[i][j] = w_t[i] * S[i][j] + k_t[i] * v_t[j]        ("Recurrent state update and output":
 *                                                          the state is the decayed sum of
 *                                                          past outer products k_i^T v_i)
 *
 * Optionally y is passed through LayerNorm over the concatenation of all H heads of a
 * token (d_model = H*D), as Finch-C2 uses in place of per-head GroupNorm:
 *     y <- (y - mean) / sqrt(var + eps) * gamma + beta,  var the biased variance.
 *
 * Conventions shared by every entry point
 *  - Pointers r, k, v, omega, u, state*, y, gamma, beta, workspace are DEVICE pointers on
 *    the current CUDA device; the caller owns every buffer.  The library never allocates
 *    device memory, keeps no global mutable state (two exceptions: the built-in scratch of
 *    wkv6_prefill_static, and the two side streams per device that the bf16 backward
 *    entry points create on first use) and, apart from wkv6_workspace_status and
 *    wkv6_prefill_static_status, never synchronises, so calls on different streams with
 *    different workspaces are independent.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; a device-side fault surfaces as a CUDA error at the caller's
 *    next synchronisation.  The bf16 backward entry points fork part of their work onto
 *    their side streams through events recorded on `stream` and join it back the same way
 *    before they return: to the caller the call is ordered on `stream` like any other.
 *  - Arguments are validated before anything is launched; on any error nothing is
 *    launched and no output is touched.
 *  - Layouts are row-major and dense:
 *        r, k, v, omega, y : [B][T][H][D] (prefill) or [B][H][D] (decode), dtype `io`
 *        u                 : [H][D] fp32
 *        state             : [B][H][D][D] fp32, state[b][h][i][j]
 *        gamma, beta       : [H*D] fp32
 *  - All pointers must be 16-byte aligned.  y must not overlap r, k, v, omega, u or the
 *    states.  state_out may equal state_in (in-place), but may not partially overlap it.
 *  - omega is the decay logit d_t; the library forms w = exp(-exp(omega)) itself.
 */
#ifndef GOLDWKV_H
#define GOLDWKV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum wkv_status {
    WKV_OK = 0,
    WKV_ERR_INVALID_ARG = 1,   /* null / misaligned / overlapping pointer, negative size   */
    WKV_ERR_UNSUPPORTED = 2,   /* D != 64, or a dtype / option combination not built      */
    WKV_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed             */
    WKV_ERR_TIMEOUT = 4,       /* a bounded device-side wait expired                       */
    WKV_ERR_WORKSPACE = 5      /* workspace missing or smaller than *_workspace_bytes()   */
} wkv_status;

typedef enum wkv_dtype {
    WKV_F32 = 0,               /* fp32 r, k, v, omega and y                                */
    WKV_BF16 = 1               /* bf16 r, k, v, omega and y                                */
} wkv_dtype;

typedef enum wkv_algo {
    WKV_ALGO_AUTO = 0,         /* library picks (chunked tensor-core path where it applies) */
    WKV_ALGO_RECURRENT = 1,    /* token-by-token fp32 recurrence on CUDA cores             */
    WKV_ALGO_CHUNKED = 2,      /* chunked prefill on tcgen05 tensor cores (bf16 I/O only)  */
    WKV_ALGO_CHUNKED_LEVELS = 3 /* chunked, every chunk through the level factorisation that
                                   takes any decay (the path WKV_ALGO_CHUNKED falls back to
                                   per sequence); bf16 I/O only, slower, for testing      */
} wkv_algo;

/* LayerNorm over the H*D concatenated head outputs of each token. */
typedef struct wkv_ln {
    const float *gamma;        /* [H*D] device, fp32, required                             */
    const float *beta;         /* [H*D] device, fp32, required                             */
    float eps;                 /* added to the variance inside the square root; > 0      */
} wkv_ln;

/* Bytes of device workspace wkv6_prefill needs for these sizes (0: none).  Depends only
 * on its arguments.  Layout on the chunked path: a 4-byte device status word at offset 0
 * (256 bytes reserved), then per (b,h) a hand-off record (chunk index, and a D x D fp32
 * state) used when a sequence moves from the fast to the level-factorised kernel;
 * LayerNorm with bf16 output adds a progress word per (b,h,segment) unit and one counter
 * (256-byte aligned) and an fp32 [B][T][H][D] staging buffer at the end. */
size_t wkv6_prefill_workspace_bytes(int B, int T, int H, int D, wkv_dtype io, int with_ln,
                                    wkv_algo algo);

/*
 * Prefill: run the recurrence over T tokens for every (b,h), starting from state_in.
 * Defined by the page's state sum and readout (section 3.4, "Recurrent state update and
 * output"); the pre-fill procedure it serves is section 3.4 "Training and Inference
 * Procedures" (tokens fed through the recurrence one by one or in parallel chunks).
 *   r, k, v, omega  [B][T][H][D] io     inputs
 *   u               [H][D] fp32         bonus
 *   state_in        [B][H][D][D] fp32   or NULL for a zero initial state
 *   state_out       [B][H][D][D] fp32   final state, or NULL (not written); may == state_in
 *   y               [B][T][H][D] io     output (LayerNorm-ed when ln != NULL)
 *   B, T, H >= 0 (B, H or T == 0 is an empty problem: with T == 0 state_out receives
 *   state_in, or zeros), D == 64.
 *   ln              NULL, or LayerNorm parameters
 *   workspace       device scratch of at least wkv6_prefill_workspace_bytes(...) bytes
 *                   (may be NULL when that is 0).  On the chunked path its first 4 bytes
 *                   are a status word that must be zero before the first call (zero-fill
 *                   new workspace; see wkv6_workspace_status); other bytes are scratch.
 *   Algorithm: WKV_ALGO_AUTO takes the chunked tensor-core kernel for bf16 I/O and the
 *   fp32 recurrence for fp32 I/O.
 *   LayerNorm: the recurrence stages fp32 rows of y in the workspace.  On the chunked path
 *   with H <= 32, when the level-factorised kernel's CTAs leave room on the device, extra
 *   CTAs of the same (cooperative) launch normalise each 64-token block of a batch row as
 *   soon as all H heads have stored it, and drop the consumed staging lines from L2;
 *   otherwise (and for fp32 I/O) a second kernel normalises the staged rows.  Same results.
 * Returns WKV_OK, or an error with nothing launched (INVALID_ARG, UNSUPPORTED, WORKSPACE)
 * or WKV_ERR_CUDA if a launch failed.
 */
wkv_status wkv6_prefill(const void *r, const void *k, const void *v, const void *omega,
                        const float *u, const float *state_in, float *state_out, void *y,
                        int B, int T, int H, int D, wkv_dtype io, const wkv_ln *ln,
                        void *workspace, size_t workspace_bytes, void *stream);

/* As wkv6_prefill, with the algorithm chosen by the caller (WKV_ALGO_CHUNKED on fp32 I/O
 * returns WKV_ERR_UNSUPPORTED). */
wkv_status wkv6_prefill_algo(const void *r, const void *k, const void *v, const void *omega,
                             const float *u, const float *state_in, float *state_out, void *y,
                             int B, int T, int H, int D, wkv_dtype io, const wkv_ln *ln,
                             wkv_algo algo, void *workspace, size_t workspace_bytes,
                             void *stream);

/*
 * Device status word of a workspace used by wkv6_prefill on the chunked path.  The chunked
 * kernel bounds every wait on its own copies and tensor-core work; if one expires, the CTA
 * drains its in-flight work, frees its tensor memory, returns early and sets this word.
 * Synchronises `stream`, returns WKV_ERR_TIMEOUT (and clears the word) if it was set,
 * WKV_OK otherwise.  The word must be zero before first use (zero-fill new workspace).
 */
wkv_status wkv6_workspace_status(void *workspace, void *stream);

/*
 * Splitting one sequence across devices (the state-passing form of the page's pre-fill,
 * section 3.4 "Training and Inference Procedures": the state carried from one span of
 * tokens to the next reproduces the single pass).  Rank p of P holds tokens
 * [p*T, (p+1)*T) of every (b,h) sequence:
 *   1. wkv6_segment_summary on its tokens: the state they build from a zero state, S_p,
 *      and each channel's total log2 decay over them, g_p = sum_t log2 w_t;
 *   2. exchange (S_p, g_p) between the ranks (one all-gather);
 *   3. wkv6_segment_carry: the state entering every segment, s_in[p + 1] =
 *      diag(2^g_p) s_in[p] + S_p from the sequence's initial state s_in[0];
 *   4. wkv6_prefill of its tokens from s_in[p].
 *
 * wkv6_segment_summary: k, v, omega [B][T][H][D] bf16 (as for wkv6_prefill; c2 != 0 takes
 * Finch-C2's normalised key k (1 - w)), T a multiple of 64 (chunk-aligned segments; else
 * WKV_ERR_UNSUPPORTED).  Outputs s_loc [B][H][D][D] fp32 and log2_decay [B][H][D] fp32.
 * Workspace: wkv6_segment_summary_workspace_bytes(...) bytes whose first word is the status
 * word of wkv6_workspace_status (zero-fill new workspace).  Runs on the tensor cores with
 * factors <= 1 only, so any decay is taken.  T == 0 writes the zero state and no decay.
 */
size_t wkv6_segment_summary_workspace_bytes(int B, int T, int H, int D);
wkv_status wkv6_segment_summary(const void *k, const void *v, const void *omega, int c2,
                                float *s_loc, float *log2_decay, int B, int T, int H, int D,
                                wkv_dtype io, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * wkv6_segment_carry: P segments' summaries laid out segment-major, s_loc [P][B][H][D][D]
 * and log2_decay [P][B][H][D] (rank p's in slot p, as an all-gather leaves them), and the
 * sequence's initial state state0 [B][H][D][D] (NULL: zero).  Writes s_in [P + 1][B][H][D][D]:
 * s_in[0] = state0, s_in[p + 1] = 2^log2_decay[p] (rows) * s_in[p] + s_loc[p] -- the state
 * entering segment p, and s_in[P] the state after the last.  fp32; no workspace.
 */
wkv_status wkv6_segment_carry(const float *state0, const float *s_loc, const float *log2_decay,
                              float *s_in, int P, int B, int H, int D, void *stream);

/* Bytes of device workspace wkv6_decode_step needs (non-zero only with LayerNorm): a block
 * of B row counters (256-byte aligned size), then, with bf16 I/O, B*H*D fp32 outputs. */
size_t wkv6_decode_workspace_bytes(int B, int H, int D, wkv_dtype io, int with_ln);

/*
 * One autoregressive step (T = 1) for every (b,h), the state updated IN PLACE: the O(1)
 * per-token recurrent update of section 3.4 "Training and Inference Procedures"
 * (autoregressive generation) applied to the recurrence above.
 *   r, k, v, omega  [B][H][D] io;  u [H][D] fp32;  state [B][H][D][D] fp32 (read, then
 *   overwritten with the new state);  y [B][H][D] io (LayerNorm-ed when ln != NULL).
 *   workspace: at least wkv6_decode_workspace_bytes(...) bytes (none without LayerNorm).
 * One kernel launch, LayerNorm included: the last CTA of each batch row to finish
 * normalises the row.  With LayerNorm the workspace's row counters (its first bytes) must
 * be zero before the first call on it (zero-fill new workspace); every call leaves them
 * zero, so one workspace serves any number of steps, in stream order.
 */
wkv_status wkv6_decode_step(const void *r, const void *k, const void *v, const void *omega,
                            const float *u, float *state, void *y, int B, int H, int D,
                            wkv_dtype io, const wkv_ln *ln, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Finch-C2's exact time mixing (GoldFinch review page, section 3.4: "Key computation with
 * normalization property" and "Receptance, value, and the new second value"; final output
 * "LayerNorm(concat(r_t . wkv_t + u'_t))").  Against the recurrence at the top of this file,
 * two things change:
 *     S[i][j] = w_t[i] S[i][j] + k_t[i] (1 - w_t[i]) v_t[j]   (the key is normalised by 1 - w)
 *     y_t[j]  = sum_i r_t[i] S[i][j] + u'_t[j]                  (no static bonus u; the second
 *                                                                value u' is added instead)
 * and LayerNorm, when requested, applies to that sum.  k is the key before the (1 - w)
 * factor; the library forms 1 - w = -expm1(-exp(omega)) itself.
 *
 * wkv6c2_prefill: as wkv6_prefill (WKV_ALGO_AUTO, same workspace query, same layouts and
 * errors) with `uprime` in place of `u`:
 *   uprime  [B][T][H][D] io  the second value u'_t of every token; required when B, T, H > 0;
 *           must not overlap y or the states.
 */
wkv_status wkv6c2_prefill(const void *r, const void *k, const void *v, const void *omega,
                          const void *uprime, const float *state_in, float *state_out, void *y,
                          int B, int T, int H, int D, wkv_dtype io, const wkv_ln *ln,
                          void *workspace, size_t workspace_bytes, void *stream);

/* wkv6c2_decode_step: as wkv6_decode_step with uprime [B][H][D] io in place of u. */
wkv_status wkv6c2_decode_step(const void *r, const void *k, const void *v, const void *omega,
                              const void *uprime, float *state, void *y, int B, int H, int D,
                              wkv_dtype io, const wkv_ln *ln, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Base Finch's own output stage, which Finch-C2 removes (GoldFinch review page, section 3.4
 * "Finch-C2 Time Mixing": modification (1) removes the gate, (2) replaces the per-head
 * GroupNorm with the full-width LayerNorm).  After the base recurrence at the top of this
 * file, each head's D outputs of each token are normalised on their own and then multiplied
 * by the gate:
 *     y[b][t][h][c] <- ((y - mean_bth) / sqrt(var_bth + eps) * gamma[h*D + c]
 *                       + beta[h*D + c]) * gate[b][t][h][c]
 * mean / var (biased) over the D = 64 channels of head h of token (b,t).  The gate is an
 * input: whatever activation produced it (the pages do not print the gate's form) is
 * applied by the caller.
 */
typedef struct wkv_gn {
    const float *gamma;        /* [H*D] device, fp32, required                             */
    const float *beta;         /* [H*D] device, fp32, required                             */
    float eps;                 /* added to the variance inside the square root; > 0      */
    const void *gate;          /* device, dtype `io`, layout of y ([B][T][H][D] prefill,
                                  [B][H][D] decode); NULL = no gate.  Must not overlap y,
                                  the states or the workspace.                            */
} wkv_gn;

/*
 * wkv6_prefill_gn: as wkv6_prefill (WKV_ALGO_AUTO; same layouts, aliasing rules and errors)
 * with the GroupNorm + gate output stage above in place of LayerNorm.  gn is required.
 * Workspace: wkv6_prefill_workspace_bytes(B, T, H, D, io, 1, WKV_ALGO_AUTO) -- the same as
 * with LayerNorm.  With bf16 I/O (the chunked path) the stage runs inside the recurrence
 * kernels, as each chunk's output is formed (a head's 64 channels are one CTA's), and the
 * workspace's LayerNorm staging area is left unused; the fp32 recurrence normalises in a
 * second kernel over fp32 rows.
 */
wkv_status wkv6_prefill_gn(const void *r, const void *k, const void *v, const void *omega,
                           const float *u, const float *state_in, float *state_out, void *y,
                           int B, int T, int H, int D, wkv_dtype io, const wkv_gn *gn,
                           void *workspace, size_t workspace_bytes, void *stream);

/* wkv6_decode_step_gn: as wkv6_decode_step with the GroupNorm + gate output stage (gn
 * required; gate [B][H][D] io or NULL), in the same kernel (each head is normalised by the
 * CTA that computes it).  No workspace is needed (workspace may be NULL); one of
 * wkv6_decode_workspace_bytes(B, H, D, io, 1) bytes is accepted. */
wkv_status wkv6_decode_step_gn(const void *r, const void *k, const void *v, const void *omega,
                               const float *u, float *state, void *y, int B, int H, int D,
                               wkv_dtype io, const wkv_gn *gn, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * Backward pass of the base recurrence (wkv6_prefill without LayerNorm) for training: the
 * gradients of a loss L with respect to every input, given dy = dL/dy and, optionally,
 * dstate_out = dL/dstate_out.  Training with all tokens in parallel is section 3.4
 * "Training and Inference Procedures" of the GoldFinch review page; the gradients are
 * the chain rule applied to the recurrence at the top of this file (G the gradient of the
 * state after token t, G = dstate_out after the last token):
 *     dr_t = S_{t-1} dy_t + u * k_t (v_t . dy_t)        dk_t = G v_t + u * r_t (v_t . dy_t)
 *     dv_t = G^T k_t + (r_t . (u * k_t)) dy_t           du   = sum_{b,t} r_t * k_t (v_t . dy_t)
 *     domega_t[i] = (sum_j G[i][j] S_{t-1}[i][j]) * w_t[i] * (-exp(omega_t[i]))
 *     G <- diag(w_t) G + r_t^T dy_t,   dstate_in = G before the first token.
 * With bf16 I/O all three run on the tensor cores, chunk by chunk: dr as the readout of the
 * forward state S_{t-1} with dy as the query, dk as the same readout of G in reversed time
 * (query v, key r, value dy), dv as the forward recurrence in reversed time with r and k
 * swapped and dy as the value (the chunked prefill on time-reversed copies); the decay
 * gradient is the equivalent sum of the pair terms that straddle each token.  A (b,h) with
 * a chunk whose decays the dr or dk pass cannot factor (a channel's decay over 64 tokens
 * below e^-60) is redone by token-by-token scans on CUDA cores in fp32, which also serve
 * fp32 I/O (with dv as a third scan).
 *   r, k, v, omega, u, state_in   the forward call's inputs (state_in NULL = zeros)
 *   dy          [B][T][H][D] io   gradient of y
 *   dstate_out  [B][H][D][D] fp32 gradient of the final state, or NULL (zero)
 *   dr, dk, dv, domega [B][T][H][D] io   outputs
 *   du          [H][D] fp32       output, summed over batch and tokens (overwritten)
 *   dstate_in   [B][H][D][D] fp32 output, or NULL (not computed)
 *   workspace   at least wkv6_backward_workspace_bytes(...) bytes; no initial contents needed.
 * No output may overlap an input, another output or the workspace.  T = 0: du = 0 and
 * dstate_in = dstate_out (or zero).  The bf16 tensor-core passes use bounded waits; if one
 * expired (a device that stopped making progress for about a second), the gradients are
 * invalid and the call does not report it (the status word is internal to the workspace).
 */
size_t wkv6_backward_workspace_bytes(int B, int T, int H, int D, wkv_dtype io);

wkv_status wkv6_backward(const void *r, const void *k, const void *v, const void *omega,
                         const float *u, const float *state_in, const void *dy,
                         const float *dstate_out, void *dr, void *dk, void *dv, void *domega,
                         float *du, float *dstate_in, int B, int T, int H, int D, wkv_dtype io,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward pass of Finch-C2's exact form (wkv6c2_prefill without LayerNorm): gradients of a
 * loss with respect to r, k, v, omega, u' and state_in, given dy and (optionally)
 * dstate_out.  With kn_t = k_t (1 - w_t) and G as for wkv6_backward:
 *     dr_t = S_{t-1} dy_t;   dkn = G v_t, dk_t = dkn (1 - w_t);   dv_t = G^T kn_t;
 *     domega_t = (sum_j G[i][j] S_{t-1}[i][j] - dkn k_t) w_t (-exp(omega_t));   du'_t = dy_t
 * (no bonus; u' enters y additively).  With bf16 I/O all three run on the tensor cores as
 * in wkv6_backward: kn formed in the dr pass; dk, Q and the direct term dkn k w from the dk
 * pass's readout dkn; dv through the chunked prefill on time-reversed copies with the query
 * k (1 - w) formed inside; the same per-(b,h) fallback to token-by-token scans on CUDA
 * cores, which also serve fp32 I/O (fp32, fp64 row scans with fp32 I/O).  The decay
 * gradient goes through the pair identity with the normalised keys.
 *   duprime  [B][T][H][D] io: output (a copy of dy), or NULL (not written).
 * Other arguments, layouts and errors as wkv6_backward; workspace: at least
 * wkv6c2_backward_workspace_bytes(...) bytes.
 */
size_t wkv6c2_backward_workspace_bytes(int B, int T, int H, int D, wkv_dtype io);

wkv_status wkv6c2_backward(const void *r, const void *k, const void *v, const void *omega,
                           const float *state_in, const void *dy, const float *dstate_out,
                           void *dr, void *dk, void *dv, void *domega, void *duprime,
                           float *dstate_in, int B, int T, int H, int D, wkv_dtype io,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * GOLD key compression and TokenCat decompression (GoldFinch review page, section 3.4
 * "GOLD Key Compression and TokenCat Decompression"): the output x_t of the last Finch-C2
 * layer is compressed by one global matrix W_KD (D x Dc, Dc = D/16 in the page's model)
 * into the cache entry c_t = x_t W_KD; a GOLD layer rebuilds the proto-key
 *     k^D_t = RMSNorm(concat(x0_t, c_t) W_KU),   W_KU (D + Dc) x D,
 * x0_t the token's input embedding, RMSNorm(z) = z / sqrt(mean(z^2) + eps) * gamma.
 * All tensors bf16 row-major except gamma (fp32); the weights are passed as the rows of
 * each linear map (the layout of a linear layer's weight, [out][in]):
 *   x, x0 [N][D];  c [N][Dc];  kd [N][D];  w_kd [Dc][D] (w_kd[j][i] = W_KD[i][j]);
 *   w_ku [D][D + Dc] (w_ku[o][i] = W_KU[i][o]);  gamma [D] fp32 or NULL (= 1).
 * The products run on the tensor cores in the library's own tcgen05 GEMM, with fp32
 * accumulation (c is rounded to bf16 once); decompression reads x0 and c in place (no
 * concatenated copy) and, for D <= 2048, applies RMSNorm to the fp32 product inside the
 * same kernel (the CTAs of a row block exchange their partial sums of squares); wider D
 * writes the fp32 product to the workspace and normalises it in a second kernel.  D and
 * Dc must be multiples of 8 and D <= 16384 (else WKV_ERR_UNSUPPORTED), N <= 2^31 - 1.
 * Outputs may not overlap inputs or the workspace.  Workspace: at least
 * gold_*_workspace_bytes(...) bytes; its first 4 bytes are a status word that the kernel
 * sets if one of its bounded waits expires (the outputs are then undefined), read and
 * cleared by wkv6_workspace_status -- zero-fill new workspace to use it.  eps must be > 0.
 */
size_t gold_compress_workspace_bytes(long N, int D, int Dc);
wkv_status gold_compress(const void *x, const void *w_kd, void *c, long N, int D, int Dc,
                         void *workspace, size_t workspace_bytes, void *stream);
size_t gold_decompress_workspace_bytes(long N, int D, int Dc);
wkv_status gold_decompress(const void *x0, const void *c, const void *w_ku, const float *gamma,
                           float eps, void *kd, long N, int D, int Dc, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Size of the scratch array built into the library for wkv6_prefill_static, per device. */
#define WKV6_STATIC_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * Prefill that allocates nothing and takes no workspace argument.  The pages have no
 * counterpart: this is a calling convention of this library, not part of the method.
 *
 * Who it is for: callers that cannot hand the library device memory at call time, for
 * example code that runs where allocating is not allowed or not safe (a runtime that
 * forbids allocation once it is running, a region whose memory is owned by someone else,
 * a latency-bound loop where an allocation might block or fail), and which also cannot
 * keep a workspace of its own alive between calls.
 *
 * Same arguments, results and errors as wkv6_prefill (WKV_ALGO_AUTO) without the two
 * workspace arguments.  The workspace wkv6_prefill would need is taken instead from a
 * scratch array of WKV6_STATIC_SCRATCH_BYTES bytes compiled into the library (one per
 * device).  Neither this call nor anything it calls allocates memory.
 *   - Limit: on the chunked path (bf16 I/O) wkv6_prefill may cut each (b,h) sequence into
 *     P segments, and its workspace grows with the number of (b,h,segment) units (about
 *     32 KB per unit).  Here P is capped: the segment count wkv6_prefill would use if its
 *     workspace fits the scratch, else the largest smaller one that fits, else P = 1 (no
 *     split; about 16 KB per (b,h), so up to 511 (b,h) pairs without LayerNorm).  A smaller
 *     P only leaves SMs idle on few-(b,h) problems; results are the same up to rounding.
 *     Sizes that do not fit even at P = 1 return WKV_ERR_WORKSPACE with nothing launched;
 *     bf16 with LayerNorm also needs 4 * B*T*H*D bytes and fits only for small problems.
 *     fp32 I/O needs no scratch.
 *   - Set-up: the first call on each device, with that device current, looks up the
 *     scratch's device address (cudaGetSymbolAddress, which may load the library's device
 *     code) and caches it with the current CUDA context; a later call in another context
 *     (for example after cudaDeviceReset) looks it up again.  A failed lookup returns
 *     WKV_ERR_CUDA.  Make that first call, on every device that will use it, before
 *     capturing a stream that will contain it.
 *   - Timeouts: the chunked kernels bound every wait; if one expires, its CTA returns early
 *     and y and state_out of that call are UNDEFINED, although the call itself returned
 *     WKV_OK (it returns before the kernels run).  The expiry is recorded in the scratch's
 *     first 4 bytes (zero when the library's device code is loaded) and stays recorded
 *     until wkv6_prefill_static_status reads and clears it.  Nothing else in the scratch
 *     has to start at zero: every other byte a call reads was written earlier in the same
 *     call.
 *   - Concurrency: all calls on one device share the one scratch.  Calls whose execution
 *     may overlap (different streams, or different host threads without ordering between
 *     them) race on it and can corrupt each other's outputs; order them (one stream, or
 *     events), or use wkv6_prefill with a workspace per stream.
 */
wkv_status wkv6_prefill_static(const void *r, const void *k, const void *v, const void *omega,
                               const float *u, const float *state_in, float *state_out, void *y,
                               int B, int T, int H, int D, wkv_dtype io, const wkv_ln *ln,
                               void *stream);

/*
 * Status of the calls to wkv6_prefill_static on the current device, as wkv6_workspace_status
 * for a caller's workspace: synchronises `stream` (order it after those calls), returns
 * WKV_ERR_TIMEOUT and clears the record if a bounded wait of one of them expired since the
 * last query (their outputs are then undefined), WKV_OK otherwise.  WKV_ERR_CUDA if the
 * scratch cannot be looked up or the copy fails.  Allocates nothing.
 */
wkv_status wkv6_prefill_static_status(void *stream);

/* Static, human-readable name of a status code. */
const char *wkv6_status_string(wkv_status s);

/* Version of this ABI (incremented on any signature change). */
int wkv6_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GOLDWKV_H */
