/*
 * TEST INFRASTRUCTURE ONLY.  Plain, slow, obviously-correct fp64 CPU oracle for the
 * Finch-C2 / RWKV-6 time-mix WKV recurrence.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load this file; the product path (libgoldwkv)
 * shares no code, header or constant with it.
 *
 * Source of the definition: "GoldFinch: High Performance RWKV/Transformer Hybrid ..."
 * review page (mlsanity.com), section 3.4, "Finch-C2 Time Mixing":
 *   - data-dependent decay        w_t = exp(-exp(d_t))             ("Data-dependent decay")
 *   - recurrent state             wkv_t = sum_{i<t} diag(prod_{j=i+1}^{t-1} w_j) k_i^T v_i
 *                                                                 ("Recurrent state update and output")
 *   - readout                     r_t . wkv_t  plus the base-Finch static bonus u
 *                                 (the bonus enters as r_t . diag(u) k_t^T v_t)
 *   - LayerNorm over the concatenation of all heads                ("... full concatenated dimension")
 *   - Finch-C2's exact form (wkv6c2_*): key k_t (1 - w_t), second value u'_t added to the
 *     readout instead of the static bonus              ("Key computation with normalization
 *                                                        property", "the new second value")
 *   - base Finch's per-head GroupNorm and output gate, which Finch-C2 removes
 *   - the backward pass of the base recurrence (the chain rule through the recursion; the
 *     page's "Training and Inference Procedures" trains all tokens in parallel)
 *   - GOLD key compression c_t = x_t W_KD and TokenCat decompression
 *     RMSNorm(concat(x0_t, c_t) W_KU)            ("GOLD Key Compression and TokenCat
 *                                                  Decompression")
 * Written in recursive form: with S_{-1} = state_in (zero if absent),
 *   y_t[j] = sum_i r_t[i] S_{t-1}[i][j] + (sum_i r_t[i] u[i] k_t[i]) v_t[j]
 *   S_t[i][j] = w_t[i] S_{t-1}[i][j] + k_t[i] v_t[j]
 * so wkv_t of the page is S_{t-1} here: the newest outer product enters undecayed and
 * w_t first touches the state when S_t is formed.  Rows of S (index i) are key/decay
 * channels, columns (index j) value channels.
 *
 * Every function here is pinned by tests/test_oracle_pins.py against brute-force sums,
 * closed forms and invariants that do not reuse this code.
 *
 * Layouts (row-major, fp64):
 *   r, k, v, omega, y : [B][T][H][D]
 *   u                 : [H][D]
 *   state_in/out      : [B][H][D][D]   (state[b][h][i][j])
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* One (b,h) sequence, tokens t0..t0+T-1, element (t,c) of a token-major tensor at
 * base[t*tstride + c]. */
static void wkv6_one_head(long T, int D, long tstride,
                          const double *r, const double *k, const double *v,
                          const double *omega, const double *u,
                          const double *s_in, double *y, double *s_out, double *S,
                          double *w)
{
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j)
            S[i * D + j] = s_in ? s_in[i * D + j] : 0.0;

    for (long t = 0; t < T; ++t) {
        const double *rt = r + t * tstride;
        const double *kt = k + t * tstride;
        const double *vt = v + t * tstride;
        const double *ot = omega + t * tstride;
        double *yt = y + t * tstride;

        /* decay of this token: w_t = exp(-exp(omega_t)) */
        for (int i = 0; i < D; ++i)
            w[i] = exp(-exp(ot[i]));

        /* bonus coefficient sum_i r_t[i] u[i] k_t[i] */
        double bonus = 0.0;
        for (int i = 0; i < D; ++i)
            bonus += rt[i] * u[i] * kt[i];

        /* readout from the state before this token */
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i)
                acc += rt[i] * S[i * D + j];
            yt[j] = acc + bonus * vt[j];
        }

        /* state update: decay rows, add the outer product k_t^T v_t */
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                S[i * D + j] = w[i] * S[i * D + j] + kt[i] * vt[j];
    }

    if (s_out)
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                s_out[i * D + j] = S[i * D + j];
}

/* Finch-C2 exact time mixing, one (b,h) sequence.  Same state and decay as above, with the
 * two changes of the page's Finch-C2 ("Key computation with normalization property" and
 * "Receptance, value, and the new second value"):
 *   - the key enters the state multiplied by (1 - w_t):  S_t = diag(w_t) S_{t-1} + (k_t (1 - w_t))^T v_t
 *   - no static bonus; a data-dependent second value u'_t is added to the readout:
 *     y_t = r_t . S_{t-1} + u'_t
 * u'_t (uprime) is token-major like y. */
static void wkv6c2_one_head(long T, int D, long tstride,
                            const double *r, const double *k, const double *v,
                            const double *omega, const double *uprime,
                            const double *s_in, double *y, double *s_out, double *S,
                            double *w)
{
    for (int i = 0; i < D; ++i)
        for (int j = 0; j < D; ++j)
            S[i * D + j] = (s_in != NULL) ? s_in[i * D + j] : 0.0;

    for (long t = 0; t < T; ++t) {
        const double *rt = r + t * tstride;
        const double *kt = k + t * tstride;
        const double *vt = v + t * tstride;
        const double *ot = omega + t * tstride;
        const double *ut = uprime + t * tstride;
        double *yt = y + t * tstride;

        for (int i = 0; i < D; ++i) {
            const double decay = exp(-exp(ot[i]));   /* w_t of this token */
            w[i] = decay;
        }

        /* readout from the state before this token, plus the second value */
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i)
                acc += S[i * D + j] * rt[i];
            yt[j] = acc + ut[j];
        }

        /* state update with the normalised key k_t (1 - w_t) */
        for (int i = 0; i < D; ++i) {
            const double kn = kt[i] * (1.0 - w[i]);
            for (int j = 0; j < D; ++j)
                S[i * D + j] = w[i] * S[i * D + j] + kn * vt[j];
        }
    }

    if (s_out)
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                s_out[i * D + j] = S[i * D + j];
}

typedef struct {
    int B, H, D;
    long T;
    const double *r, *k, *v, *omega, *u, *s_in;
    const double *uprime;   /* Finch-C2 second value [B][T][H][D], or NULL (base Finch) */
    double *y, *s_out;
    int next;               /* next (b*H+h) unit to take */
    pthread_mutex_t lock;
} job_t;

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int D = J->D;
    double *S = (double *)malloc(sizeof(double) * (size_t)D * D);
    double *w = (double *)malloc(sizeof(double) * (size_t)D);
    if (!S || !w) {
        free(S);
        free(w);
        return (void *)1;
    }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int unit = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (unit >= J->B * J->H)
            break;
        int b = unit / J->H, h = unit % J->H;
        long tstride = (long)J->H * D;
        size_t x0 = ((size_t)b * J->T * J->H + h) * D;      /* element (b, t=0, h, 0) */
        size_t s0 = ((size_t)b * J->H + h) * D * D;
        if (J->uprime)
            wkv6c2_one_head(J->T, D, tstride, J->r + x0, J->k + x0, J->v + x0, J->omega + x0,
                            J->uprime + x0, J->s_in ? J->s_in + s0 : NULL, J->y + x0,
                            J->s_out ? J->s_out + s0 : NULL, S, w);
        else
            wkv6_one_head(J->T, D, tstride, J->r + x0, J->k + x0, J->v + x0, J->omega + x0,
                          J->u + (size_t)h * D, J->s_in ? J->s_in + s0 : NULL, J->y + x0,
                          J->s_out ? J->s_out + s0 : NULL, S, w);
    }
    free(S);
    free(w);
    return NULL;
}

static int run_units(job_t *J, int nthreads)
{
    J->next = 0;
    pthread_mutex_init(&J->lock, NULL);
    if (nthreads > J->B * J->H)
        nthreads = J->B * J->H;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0, rc = 0;
    for (int n = 0; n < nthreads; ++n) {
        if (pthread_create(&tid[n], NULL, worker, J) != 0) {
            rc = -2;
            break;
        }
        ++started;
    }
    for (int n = 0; n < started; ++n) {
        void *ret = NULL;
        pthread_join(tid[n], &ret);
        if (ret)
            rc = -2;
    }
    free(tid);
    pthread_mutex_destroy(&J->lock);
    return rc;
}

/* Full prefill over [B][T][H][D] inputs.  state_in may be NULL (zeros); state_out may be
 * NULL (not written) or equal state_in.  Runs the (b,h) units on nthreads POSIX threads.
 * Returns 0 on success, -1 on bad arguments, -2 if a thread could not be started. */
int wkv6_oracle_prefill(int B, long T, int H, int D,
                        const double *r, const double *k, const double *v,
                        const double *omega, const double *u, const double *state_in,
                        double *y, double *state_out, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || D <= 0 || nthreads <= 0)
        return -1;
    if (B == 0 || H == 0)
        return 0;
    job_t J;
    J.B = B; J.T = T; J.H = H; J.D = D;
    J.r = r; J.k = k; J.v = v; J.omega = omega; J.u = u; J.s_in = state_in;
    J.uprime = NULL;
    J.y = y; J.s_out = state_out;
    return run_units(&J, nthreads);
}

/* Finch-C2 prefill (see wkv6c2_one_head): uprime [B][T][H][D] replaces u. */
int wkv6c2_oracle_prefill(int B, long T, int H, int D,
                          const double *r, const double *k, const double *v,
                          const double *omega, const double *uprime, const double *state_in,
                          double *y, double *state_out, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || D <= 0 || nthreads <= 0 || (!uprime && T > 0 && B > 0 && H > 0))
        return -1;
    if (B == 0 || H == 0)
        return 0;
    job_t J;
    J.B = B; J.T = T; J.H = H; J.D = D;
    J.r = r; J.k = k; J.v = v; J.omega = omega; J.u = NULL; J.s_in = state_in;
    J.uprime = uprime;
    J.y = y; J.s_out = state_out;
    return run_units(&J, nthreads);
}

/* One autoregressive step (T = 1) for every (b,h), state updated in place.
 * r, k, v, omega, y : [B][H][D];  state : [B][H][D][D]. */
int wkv6_oracle_decode_step(int B, int H, int D,
                            const double *r, const double *k, const double *v,
                            const double *omega, const double *u, double *state,
                            double *y, int nthreads)
{
    return wkv6_oracle_prefill(B, 1, H, D, r, k, v, omega, u, state, y, state, nthreads);
}

/* Finch-C2 autoregressive step, state updated in place. */
int wkv6c2_oracle_decode_step(int B, int H, int D,
                              const double *r, const double *k, const double *v,
                              const double *omega, const double *uprime, double *state,
                              double *y, int nthreads)
{
    return wkv6c2_oracle_prefill(B, 1, H, D, r, k, v, omega, uprime, state, y, state, nthreads);
}

/* LayerNorm of each of the N rows of x[N][C] over its C entries:
 *   out = (x - mean) / sqrt(var + eps) * gamma + beta,  var the biased (1/C) variance.
 * gamma/beta may be NULL (1 and 0).  out may equal x. */
int wkv6_oracle_layernorm(long N, int C, const double *x, const double *gamma,
                          const double *beta, double eps, double *out)
{
    if (N < 0 || C <= 0)
        return -1;
    for (long n = 0; n < N; ++n) {
        const double *xr = x + n * (long)C;
        double *orow = out + n * (long)C;
        double mean = 0.0;
        for (int c = 0; c < C; ++c)
            mean += xr[c];
        mean /= (double)C;
        double var = 0.0;
        for (int c = 0; c < C; ++c)
            var += (xr[c] - mean) * (xr[c] - mean);
        var /= (double)C;
        double inv = 1.0 / sqrt(var + eps);
        for (int c = 0; c < C; ++c) {
            double g = gamma ? gamma[c] : 1.0;
            double bb = beta ? beta[c] : 0.0;
            orow[c] = (xr[c] - mean) * inv * g + bb;
        }
    }
    return 0;
}

/* Base Finch's output normalisation, per head (the page's "per-head GroupNorm" that
 * Finch-C2 replaces by LayerNorm), followed by the output gate:
 *   out[n][h][c] = ((x[n][h][c] - mean_nh) / sqrt(var_nh + eps) * gamma[h*D + c] + beta[h*D + c])
 *                  * gate[n][h][c]
 * mean_nh / var_nh (biased) over the D channels of head h of row n; x, gate, out [N][H][D];
 * gamma / beta [H*D] may be NULL (1 / 0); gate may be NULL (1).  out may equal x. */
int wkv6_oracle_groupnorm_gate(long N, int H, int D, const double *x, const double *gamma,
                               const double *beta, double eps, const double *gate, double *out)
{
    if (N < 0 || H <= 0 || D <= 0)
        return -1;
    for (long n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            const long base = (n * H + h) * (long)D;
            double mu = 0.0;
            for (int c = 0; c < D; ++c)
                mu += x[base + c];
            mu /= (double)D;
            double s2 = 0.0;
            for (int c = 0; c < D; ++c)
                s2 += (x[base + c] - mu) * (x[base + c] - mu);
            s2 /= (double)D;
            const double rs = 1.0 / sqrt(s2 + eps);
            for (int c = 0; c < D; ++c) {
                const double ga = gamma ? gamma[h * D + c] : 1.0;
                const double be = beta ? beta[h * D + c] : 0.0;
                const double gt = gate ? gate[base + c] : 1.0;
                out[base + c] = ((x[base + c] - mu) * rs * ga + be) * gt;
            }
        }
    }
    return 0;
}


/* Backward pass of the base recurrence (wkv6_one_head) for one (b,h) sequence: the adjoint
 * of the recursion written out by the chain rule, token by token in reverse.  The forward
 * states are recomputed first and kept (Sall[t] = state before token t, t = 0..T).
 * With G the gradient with respect to the state after token t (G = dstate_out, or zero, at
 * the end of the sequence):
 *   dv_t[j]  = sum_i G[i][j] k_t[i] + (sum_i r_t[i] u[i] k_t[i]) dy_t[j]
 *   dk_t[i]  = sum_j G[i][j] v_t[j] + r_t[i] u[i] (v_t . dy_t)
 *   dr_t[i]  = sum_j Sall[t][i][j] dy_t[j] + u[i] k_t[i] (v_t . dy_t)
 *   dw_t[i]  = sum_j G[i][j] Sall[t][i][j]
 *   domega_t = dw_t * dw/domega = dw_t * (-exp(omega_t) w_t)
 *   du[i]   += r_t[i] k_t[i] (v_t . dy_t)
 *   G[i][j]  = w_t[i] G[i][j] + r_t[i] dy_t[j]   (now the gradient of the state before t)
 * and dstate_in = G at the start.  du_acc accumulates (summed over all calls). */
static void wkv6_one_head_backward(long T, int D, long tstride,
                                   const double *r, const double *k, const double *v,
                                   const double *omega, const double *u, const double *s_in,
                                   const double *dy, const double *ds_out,
                                   double *dr, double *dk, double *dv, double *domega,
                                   double *du_acc, double *ds_in, double *Sall, double *G)
{
    const long DD = (long)D * D;
    for (long e = 0; e < DD; ++e)
        Sall[e] = s_in ? s_in[e] : 0.0;
    for (long t = 0; t < T; ++t) {
        const double *kt = k + t * tstride, *vt = v + t * tstride, *ot = omega + t * tstride;
        const double *Sb = Sall + t * DD;
        double *Sa = Sall + (t + 1) * DD;
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            for (int j = 0; j < D; ++j)
                Sa[i * D + j] = wi * Sb[i * D + j] + kt[i] * vt[j];
        }
    }

    for (long e = 0; e < DD; ++e)
        G[e] = ds_out ? ds_out[e] : 0.0;
    for (long t = T - 1; t >= 0; --t) {
        const double *rt = r + t * tstride, *kt = k + t * tstride, *vt = v + t * tstride;
        const double *ot = omega + t * tstride, *dyt = dy + t * tstride;
        const double *Sprev = Sall + t * DD;          /* state before token t */
        double *drt = dr + t * tstride, *dkt = dk + t * tstride, *dvt = dv + t * tstride;
        double *dot = domega + t * tstride;

        double vdy = 0.0, rku = 0.0;
        for (int j = 0; j < D; ++j)
            vdy += vt[j] * dyt[j];
        for (int i = 0; i < D; ++i)
            rku += rt[i] * u[i] * kt[i];

        for (int j = 0; j < D; ++j) {
            double g = 0.0;
            for (int i = 0; i < D; ++i)
                g += G[i * D + j] * kt[i];
            dvt[j] = g + rku * dyt[j];
        }
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            double gk = 0.0, gr = 0.0, gw = 0.0;
            for (int j = 0; j < D; ++j) {
                gk += G[i * D + j] * vt[j];
                gr += Sprev[i * D + j] * dyt[j];
                gw += G[i * D + j] * Sprev[i * D + j];
            }
            dkt[i] = gk + rt[i] * u[i] * vdy;
            drt[i] = gr + u[i] * kt[i] * vdy;
            dot[i] = gw * (-exp(ot[i]) * wi);
            du_acc[i] += rt[i] * kt[i] * vdy;
        }
        /* carry the gradient to the state before token t */
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            for (int j = 0; j < D; ++j)
                G[i * D + j] = wi * G[i * D + j] + rt[i] * dyt[j];
        }
    }
    if (ds_in)
        for (long e = 0; e < DD; ++e)
            ds_in[e] = G[e];
}

/* Gradients of a loss L(y, state_out) with respect to every input of wkv6_oracle_prefill,
 * given dy = dL/dy [B][T][H][D] and dstate_out = dL/dstate_out [B][H][D][D] (NULL: zero).
 * Outputs dr, dk, dv, domega [B][T][H][D]; du [H][D] (summed over b and t); dstate_in
 * [B][H][D][D] (NULL: not written).  state_in NULL means zeros.  Sequential over (b,h).
 * Returns 0, -1 on bad arguments, -3 if memory for the kept states cannot be had. */
int wkv6_oracle_backward(int B, long T, int H, int D,
                         const double *r, const double *k, const double *v,
                         const double *omega, const double *u, const double *state_in,
                         const double *dy, const double *dstate_out,
                         double *dr, double *dk, double *dv, double *domega,
                         double *du, double *dstate_in)
{
    if (B < 0 || T < 0 || H < 0 || D <= 0)
        return -1;
    for (long e = 0; e < (long)H * D; ++e)
        du[e] = 0.0;
    if (B == 0 || H == 0)
        return 0;
    const long DD = (long)D * D;
    double *Sall = (double *)malloc(sizeof(double) * (size_t)(T + 1) * (size_t)DD);
    double *G = (double *)malloc(sizeof(double) * (size_t)DD);
    if (!Sall || !G) {
        free(Sall);
        free(G);
        return -3;
    }
    const long tstride = (long)H * D;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t x0 = ((size_t)b * T * H + h) * D;
            const size_t s0 = ((size_t)b * H + h) * DD;
            wkv6_one_head_backward(T, D, tstride, r + x0, k + x0, v + x0, omega + x0,
                                   u + (size_t)h * D, state_in ? state_in + s0 : NULL, dy + x0,
                                   dstate_out ? dstate_out + s0 : NULL, dr + x0, dk + x0,
                                   dv + x0, domega + x0, du + (size_t)h * D,
                                   dstate_in ? dstate_in + s0 : NULL, Sall, G);
        }
    free(Sall);
    free(G);
    return 0;
}

/* GOLD key compression (GoldFinch review page, section 3.4 "GOLD Key Compression and
 * TokenCat Decompression", compression step): c_t = x_t W_KD, W_KD a D x Dc matrix
 * (Dc = D/16 in the page's model).  W_KD is passed transposed, as the rows of the linear
 * map: w_kd[j][i] = W_KD[i][j], [Dc][D].  x [N][D], c [N][Dc]. */
int gold_oracle_compress(long N, int D, int Dc, const double *x, const double *w_kd, double *c)
{
    if (N < 0 || D <= 0 || Dc <= 0)
        return -1;
    for (long n = 0; n < N; ++n)
        for (int j = 0; j < Dc; ++j) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i)
                acc += x[n * D + i] * w_kd[(long)j * D + i];
            c[n * Dc + j] = acc;
        }
    return 0;
}

/* TokenCat decompression (same section): k^D_t = RMSNorm(concat(x0_t, c_t) W_KU), W_KU a
 * (D + Dc) x D matrix passed transposed as w_ku[o][i] = W_KU[i][o], [D][D + Dc].  RMSNorm of
 * a row z of D values: z[o] / sqrt(mean_o z[o]^2 + eps) * gamma[o] (gamma NULL = 1).
 * x0 [N][D], c [N][Dc], kd [N][D]. */
int gold_oracle_decompress(long N, int D, int Dc, const double *x0, const double *c,
                           const double *w_ku, const double *gamma, double eps, double *kd)
{
    if (N < 0 || D <= 0 || Dc <= 0 || !(eps >= 0.0))
        return -1;
    const int K = D + Dc;
    double *z = (double *)malloc(sizeof(double) * (size_t)D);
    double *cat = (double *)malloc(sizeof(double) * (size_t)K);
    if (!z || !cat) {
        free(z);
        free(cat);
        return -3;
    }
    for (long n = 0; n < N; ++n) {
        /* the concatenation [x0_t, c_t] */
        for (int i = 0; i < D; ++i)
            cat[i] = x0[n * D + i];
        for (int j = 0; j < Dc; ++j)
            cat[D + j] = c[n * Dc + j];
        double ms = 0.0;
        for (int o = 0; o < D; ++o) {
            double acc = 0.0;
            for (int i = 0; i < K; ++i)
                acc += cat[i] * w_ku[(long)o * K + i];
            z[o] = acc;
            ms += acc * acc;
        }
        ms /= (double)D;
        const double inv_rms = 1.0 / sqrt(ms + eps);
        for (int o = 0; o < D; ++o)
            kd[n * D + o] = z[o] * inv_rms * (gamma ? gamma[o] : 1.0);
    }
    free(z);
    free(cat);
    return 0;
}

/* Backward pass of Finch-C2's exact form (wkv6c2_one_head) for one (b,h) sequence, the
 * adjoint written out as for the base form.  With kn_t = k_t (1 - w_t) the normalised key
 * and G the gradient of the state after token t (dstate_out, or zero, at the end):
 *   dv_t[j]   = sum_i G[i][j] kn_t[i]                    (no bonus in this form)
 *   dkn[i]    = sum_j G[i][j] v_t[j];   dk_t[i] = dkn[i] (1 - w_t[i])
 *   dr_t[i]   = sum_j Sall[t][i][j] dy_t[j]
 *   dw_t[i]   = sum_j G[i][j] Sall[t][i][j] - dkn[i] k_t[i]    (kn depends on w too)
 *   domega_t  = dw_t (-exp(omega_t) w_t)
 *   duprime_t = dy_t                                      (u'_t is added to y_t)
 *   G[i][j]   = w_t[i] G[i][j] + r_t[i] dy_t[j]
 * and dstate_in = G at the start. */
static void wkv6c2_one_head_backward(long T, int D, long tstride,
                                     const double *r, const double *k, const double *v,
                                     const double *omega, const double *s_in,
                                     const double *dy, const double *ds_out,
                                     double *dr, double *dk, double *dv, double *domega,
                                     double *duprime, double *ds_in, double *Sall, double *G)
{
    const long DD = (long)D * D;
    for (long e = 0; e < DD; ++e)
        Sall[e] = s_in ? s_in[e] : 0.0;
    for (long t = 0; t < T; ++t) {
        const double *kt = k + t * tstride, *vt = v + t * tstride, *ot = omega + t * tstride;
        const double *Sb = Sall + t * DD;
        double *Sa = Sall + (t + 1) * DD;
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            const double kni = kt[i] * (1.0 - wi);
            for (int j = 0; j < D; ++j)
                Sa[i * D + j] = wi * Sb[i * D + j] + kni * vt[j];
        }
    }

    for (long e = 0; e < DD; ++e)
        G[e] = ds_out ? ds_out[e] : 0.0;
    for (long t = T - 1; t >= 0; --t) {
        const double *rt = r + t * tstride, *kt = k + t * tstride, *vt = v + t * tstride;
        const double *ot = omega + t * tstride, *dyt = dy + t * tstride;
        const double *Sprev = Sall + t * DD;
        double *drt = dr + t * tstride, *dkt = dk + t * tstride, *dvt = dv + t * tstride;
        double *dot = domega + t * tstride, *dut = duprime + t * tstride;

        for (int j = 0; j < D; ++j) {
            double g = 0.0;
            for (int i = 0; i < D; ++i)
                g += G[i * D + j] * (kt[i] * (1.0 - exp(-exp(ot[i]))));
            dvt[j] = g;
            dut[j] = dyt[j];
        }
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            double gkn = 0.0, gr = 0.0, gw = 0.0;
            for (int j = 0; j < D; ++j) {
                gkn += G[i * D + j] * vt[j];
                gr += dyt[j] * Sprev[i * D + j];
                gw += Sprev[i * D + j] * G[i * D + j];
            }
            dkt[i] = gkn * (1.0 - wi);
            drt[i] = gr;
            dot[i] = (gw - gkn * kt[i]) * (-exp(ot[i]) * wi);
        }
        for (int i = 0; i < D; ++i) {
            const double wi = exp(-exp(ot[i]));
            for (int j = 0; j < D; ++j)
                G[i * D + j] = G[i * D + j] * wi + rt[i] * dyt[j];
        }
    }
    if (ds_in)
        for (long e = 0; e < DD; ++e)
            ds_in[e] = G[e];
}

/* Gradients of a loss L(y, state_out) with respect to every input of wkv6c2_oracle_prefill
 * (r, k, v, omega, uprime, state_in), given dy and dstate_out (NULL: zero).  Outputs
 * dr, dk, dv, domega, duprime [B][T][H][D]; dstate_in [B][H][D][D] (NULL: not written).
 * Returns 0, -1 on bad arguments, -3 if memory for the kept states cannot be had. */
int wkv6c2_oracle_backward(int B, long T, int H, int D,
                           const double *r, const double *k, const double *v,
                           const double *omega, const double *state_in,
                           const double *dy, const double *dstate_out,
                           double *dr, double *dk, double *dv, double *domega,
                           double *duprime, double *dstate_in)
{
    if (B < 0 || T < 0 || H < 0 || D <= 0)
        return -1;
    if (B == 0 || H == 0)
        return 0;
    const long DD = (long)D * D;
    double *Sall = (double *)malloc(sizeof(double) * (size_t)(T + 1) * (size_t)DD);
    double *G = (double *)malloc(sizeof(double) * (size_t)DD);
    if (!Sall || !G) {
        free(Sall);
        free(G);
        return -3;
    }
    const long tstride = (long)H * D;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t x0 = ((size_t)b * T * H + h) * D;
            const size_t s0 = ((size_t)b * H + h) * DD;
            wkv6c2_one_head_backward(T, D, tstride, r + x0, k + x0, v + x0, omega + x0,
                                     state_in ? state_in + s0 : NULL, dy + x0,
                                     dstate_out ? dstate_out + s0 : NULL, dr + x0, dk + x0,
                                     dv + x0, domega + x0, duprime + x0,
                                     dstate_in ? dstate_in + s0 : NULL, Sall, G);
        }
    free(Sall);
    free(G);
    return 0;
}
