"""Independent checks ("pins") of the fp64 oracle.

None of these reuses the oracle's loop: each computes the expected result from another
statement of the method on the GoldFinch review page, section 3.4 "Finch-C2 Time Mixing",
or from mathematics that the definition fixes:

* explicit_sum      - the page's state as an explicit sum over past tokens of
                      diag(prod_{j=i+1}^{t-1} w_j) k_i^T v_i ("Recurrent state update and
                      output"), products formed one by one, O(T^3 D) brute force;
* t1_closed_form    - a single token: y = (r.(u*k)) v + r S0, S1 = diag(w) S0 + k^T v;
* decode_closed_form- the same closed form through the decode entry point;
* linear_attention  - w == 1 and u = 0 is strictly causal linear attention
                      ("Transformers are RNNs", cited on the citation-graph page):
                      y = tril(R K^T, -1) V + R S0;
* zero_decay        - w == 0 keeps one token of memory:
                      y_t = (r_t.(u*k_t)) v_t + (r_t.k_{t-1}) v_{t-1},  S_T = k_{T-1}^T v_{T-1};
* geometric         - per-channel constant decay with constant k, v from zero state:
                      S_t[i][j] = k_i v_j (1 - w_i^t) / (1 - w_i)  (geometric series);
* split_carry       - O(1)-per-token state passing: running [0, t1) then [t1, T) from the
                      carried state equals the full run, for several t1;
* linearity         - y and S are jointly linear in (v, S0), y is linear in r;
* ln_moments        - LayerNorm output has mean 0 and variance var/(var+eps);
* ln_torch          - LayerNorm equals torch.nn.functional.layer_norm in fp64;
* ln_shift          - LayerNorm is invariant to adding a constant to every channel.

Finch-C2's exact form (key k_t (1 - w_t), second value u'_t instead of the static bonus;
section 3.4 "Key computation with normalization property" and "the new second value"):

* c2_explicit_sum   - the explicit sum with the normalised keys, brute force, plus u'_t;
* c2_normalised_rows- the property the page gives for k (1 - w): with k = v = 1 and every
                      state row starting at 1, each row stays exactly 1 for any decays
                      (S_t = w S_{t-1} + (1 - w) 1), so y_t = sum_i r_t[i] + u'_t;
* c2_second_value   - y is affine in u' with unit slope and the state does not see u';
* c2_decode         - the decode step's closed form with the normalised key.

Base Finch's per-head GroupNorm and output gate:

* gn_moments        - every head of every row has mean 0 and variance var/(var+eps) before
                      the affine part;
* gn_torch          - GroupNorm equals torch.nn.functional.group_norm (H groups over H*D
                      channels) in fp64;
* gn_gate           - the gate multiplies the normalised output elementwise (gate 1 and
                      gate 2x give x and 2x, a random gate gives the product);
* gn_head_local     - changing one head's inputs changes only that head's outputs.

The backward pass (gradients of a loss sum(y * dy) + sum(S_T * dS_T) with respect to r, k,
v, omega, u and the initial state):

* bwd_finite_diff   - central finite differences of that loss through the (pinned) forward
                      entry point, every input element one by one, on tiny sizes;
* bwd_autograd      - torch autograd through an independent torch statement of the
                      explicit-sum form (products formed one by one), fp64;
* bwd_decay_identity- the decay gradient equals the sum of the pair terms that straddle the
                      token, which rearranges to
                      dlog w_t = <S_T, dS_T>_row + sum_{s>t} r_s dr_s' - sum_{s>=t} k_s dk_s'
                      (dr', dk' without their bonus parts): a relation between outputs;
* bwd_empty         - T = 0: dS_0 = dS_T and every other gradient is zero.
* c2_bwd_finite_diff- Finch-C2's backward against central differences through the C2
                      forward entry point (inputs r, k, v, omega, u', S_0);
* c2_bwd_autograd   - Finch-C2's backward against torch autograd through an independent
                      torch statement of the C2 explicit sum;
* c2_bwd_decay_identity - the pair identity with the normalised keys as sources
                      (Q_s = kn_s dkn_s, dkn = dk / (1 - w)), plus kn's own dependence on w:
                      domega_t = -exp(omega_t) (dlog w_t - dkn_t k_t w_t).

GOLD key compression and TokenCat decompression (section 3.4 "GOLD Key Compression and
TokenCat Decompression"):

* gold_compress_matmul  - c = x W_KD equals numpy's matrix product;
* gold_decompress_blocks- concat(x0, c) W_KU equals x0 W_KU[:D] + c W_KU[D:] (numpy), then
                          an RMSNorm written out in numpy;
* gold_rmsnorm_torch    - the same through torch.nn.functional.rms_norm, with a large eps;
* gold_scale_invariance - with eps = 0, scaling x0 and c by any a > 0 leaves the output
                          unchanged, and every row of output / gamma has mean square 1.

``run_all(oracle)`` returns the list of failing pin names; the mutation test uses it to
show that plausible mistakes planted in the oracle are caught.
"""
from __future__ import annotations

import numpy as np
import torch

RTOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, B, T, H, D, omega=(-6.0, 1.0), s0=True):
    g = _rng(seed)
    r = g.normal(0, 0.3, (B, T, H, D))
    k = g.normal(0, 0.3, (B, T, H, D))
    v = g.normal(0, 0.3, (B, T, H, D))
    om = g.uniform(omega[0], omega[1], (B, T, H, D))
    u = g.normal(0, 0.5, (H, D))
    S0 = g.normal(0, 0.1, (B, H, D, D)) if s0 else np.zeros((B, H, D, D))
    return r, k, v, om, u, S0


def _close(a, b, rtol=RTOL):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(1e-300, float(np.max(np.abs(b))) if b.size else 1.0)
    return a.shape == b.shape and float(np.max(np.abs(a - b))) <= rtol * scale if a.size else True


def brute_force_explicit(r, k, v, om, u, S0):
    """y and final state from the explicit-sum form, every product taken one by one."""
    B, T, H, D = r.shape
    w = np.exp(-np.exp(om))
    y = np.zeros_like(r)
    S_fin = np.zeros((B, H, D, D))
    for b in range(B):
        for h in range(H):
            for t in range(T + 1):
                # wkv_t: state seen by token t (t == T gives the final state)
                wkv = np.zeros((D, D))
                decay0 = np.ones(D)
                for j in range(0, t):
                    decay0 = decay0 * w[b, j, h]
                wkv = wkv + decay0[:, None] * S0[b, h]
                for i in range(0, t):
                    dec = np.ones(D)
                    for j in range(i + 1, t):
                        dec = dec * w[b, j, h]
                    wkv = wkv + (dec * k[b, i, h])[:, None] * v[b, i, h][None, :]
                if t < T:
                    rt = r[b, t, h]
                    bonus = float(np.sum(rt * u[h] * k[b, t, h]))
                    y[b, t, h] = rt @ wkv + bonus * v[b, t, h]
                else:
                    S_fin[b, h] = wkv
    return y, S_fin


def pin_explicit_sum(o):
    ok = True
    for seed, (B, T, H, D), s0 in [(1, (2, 9, 2, 8), True), (2, (1, 6, 1, 64), True),
                                   (3, (1, 12, 3, 4), False)]:
        r, k, v, om, u, S0 = _inputs(seed, B, T, H, D, s0=s0)
        y, S = o.prefill(r, k, v, om, u, S0)
        ye, Se = brute_force_explicit(r, k, v, om, u, S0)
        ok &= _close(y, ye) and _close(S, Se)
    return ok


def pin_t1_closed_form(o):
    r, k, v, om, u, S0 = _inputs(4, 3, 1, 2, 16)
    y, S = o.prefill(r, k, v, om, u, S0)
    w = np.exp(-np.exp(om[:, 0]))
    ok = True
    for b in range(3):
        for h in range(2):
            rr, kk, vv = r[b, 0, h], k[b, 0, h], v[b, 0, h]
            y_ref = np.dot(rr * u[h], kk) * vv + rr @ S0[b, h]
            S_ref = np.diag(w[b, h]) @ S0[b, h] + np.outer(kk, vv)
            ok &= _close(y[b, 0, h], y_ref) and _close(S[b, h], S_ref)
    return ok


def pin_decode_closed_form(o):
    g = _rng(5)
    B, H, D = 4, 3, 64
    r, k, v = (g.normal(0, 0.3, (B, H, D)) for _ in range(3))
    om = g.uniform(-6, 1, (B, H, D))
    u = g.normal(0, 0.5, (H, D))
    S0 = g.normal(0, 0.1, (B, H, D, D))
    y, S = o.decode_step(r, k, v, om, u, S0)
    w = np.exp(-np.exp(om))
    y_ref = np.einsum("bhi,hi,bhi->bh", r, u, k)[..., None] * v + np.einsum("bhi,bhij->bhj", r, S0)
    S_ref = w[..., None] * S0 + k[..., :, None] * v[..., None, :]
    return _close(y, y_ref) and _close(S, S_ref)


def pin_linear_attention(o):
    r, k, v, _, _, S0 = _inputs(6, 2, 33, 2, 16)
    om = np.full_like(r, -60.0)          # exp(-exp(-60)) == 1.0 in fp64
    assert np.all(np.exp(-np.exp(om)) == 1.0)
    u = np.zeros((2, 16))
    y, S = o.prefill(r, k, v, om, u, S0)
    ok = True
    for b in range(2):
        for h in range(2):
            R, K, V = r[b, :, h], k[b, :, h], v[b, :, h]
            y_ref = np.tril(R @ K.T, -1) @ V + R @ S0[b, h]
            S_ref = S0[b, h] + K.T @ V
            ok &= _close(y[b, :, h], y_ref) and _close(S[b, h], S_ref)
    return ok


def pin_zero_decay(o):
    r, k, v, _, u, S0 = _inputs(7, 2, 20, 2, 16)
    om = np.full_like(r, 8.0)            # exp(-exp(8)) == 0.0 in fp64
    assert np.all(np.exp(-np.exp(om)) == 0.0)
    y, S = o.prefill(r, k, v, om, u, S0)
    ok = True
    for b in range(2):
        for h in range(2):
            R, K, V = r[b, :, h], k[b, :, h], v[b, :, h]
            bonus = np.sum(R * u[h] * K, axis=1)
            y_ref = bonus[:, None] * V
            y_ref[0] += R[0] @ S0[b, h]
            y_ref[1:] += np.sum(R[1:] * K[:-1], axis=1)[:, None] * V[:-1]
            ok &= _close(y[b, :, h], y_ref) and _close(S[b, h], np.outer(K[-1], V[-1]))
    return ok


def pin_geometric(o):
    g = _rng(8)
    T, H, D = 50, 2, 16
    om_c = g.uniform(-3, 0.5, (H, D))
    k_c = g.normal(0, 0.3, (H, D))
    v_c = g.normal(0, 0.3, (H, D))
    r = g.normal(0, 0.3, (1, T, H, D))
    u = g.normal(0, 0.5, (H, D))
    om = np.broadcast_to(om_c, (1, T, H, D)).copy()
    k = np.broadcast_to(k_c, (1, T, H, D)).copy()
    v = np.broadcast_to(v_c, (1, T, H, D)).copy()
    y, S = o.prefill(r, k, v, om, u, None)
    w = np.exp(-np.exp(om_c))
    ok = True
    for h in range(H):
        geo_T = (1 - w[h] ** T) / (1 - w[h])
        ok &= _close(S[0, h], (k_c[h] * geo_T)[:, None] * v_c[h][None, :])
        for t in range(T):
            geo_t = (1 - w[h] ** t) / (1 - w[h])
            y_ref = np.dot(r[0, t, h], k_c[h] * geo_t) * v_c[h] + np.dot(r[0, t, h] * u[h], k_c[h]) * v_c[h]
            ok &= _close(y[0, t, h], y_ref)
    return ok


def pin_split_carry(o):
    r, k, v, om, u, S0 = _inputs(9, 2, 40, 2, 16)
    y, S = o.prefill(r, k, v, om, u, S0)
    ok = True
    for t1 in (1, 17, 20, 39):
        y1, S1 = o.prefill(r[:, :t1], k[:, :t1], v[:, :t1], om[:, :t1], u, S0)
        y2, S2 = o.prefill(r[:, t1:], k[:, t1:], v[:, t1:], om[:, t1:], u, S1)
        ok &= _close(np.concatenate([y1, y2], axis=1), y, 1e-12) and _close(S2, S, 1e-12)
    return ok


def pin_linearity(o):
    r, k, v1, om, u, S1 = _inputs(10, 2, 25, 2, 16)
    _, _, v2, _, _, S2 = _inputs(11, 2, 25, 2, 16)
    ya, Sa = o.prefill(r, k, v1, om, u, S1)
    yb, Sb = o.prefill(r, k, v2, om, u, S2)
    yc, Sc = o.prefill(r, k, v1 + v2, om, u, S1 + S2)
    yd, _ = o.prefill(2.5 * r, k, v1, om, u, S1)
    return _close(yc, ya + yb, 1e-12) and _close(Sc, Sa + Sb, 1e-12) and _close(yd, 2.5 * ya, 1e-12)


def pin_ln_moments(o):
    g = _rng(12)
    x = g.normal(0.3, 2.0, (7, 96))
    eps = 1e-5
    out = o.layernorm(x, None, None, eps)
    var_x = x.var(axis=1)
    return (float(np.max(np.abs(out.mean(axis=1)))) < 1e-12 and
            _close(out.var(axis=1), var_x / (var_x + eps), 1e-12))


def pin_ln_torch(o):
    g = _rng(13)
    x = g.normal(0.0, 1.5, (5, 3, 64))
    gam = 1.0 + 0.1 * g.normal(size=64)
    bet = 0.1 * g.normal(size=64)
    out = o.layernorm(x, gam, bet, 1e-5)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (64,), torch.from_numpy(gam),
                                         torch.from_numpy(bet), 1e-5).numpy()
    return _close(out, ref, 1e-12)


def pin_ln_shift(o):
    g = _rng(14)
    x = g.normal(0.0, 1.0, (6, 128))
    gam = 1.0 + 0.1 * g.normal(size=128)
    bet = 0.1 * g.normal(size=128)
    a = o.layernorm(x, gam, bet, 1e-5)
    b = o.layernorm(x + 3.25, gam, bet, 1e-5)
    return _close(a, b, 1e-10)


def pin_c2_explicit_sum(o):
    ok = True
    for seed, (B, T, H, D), s0 in [(11, (2, 8, 2, 8), True), (12, (1, 6, 1, 64), False)]:
        r, k, v, om, _, S0 = _inputs(seed, B, T, H, D, s0=s0)
        up = _rng(seed + 100).normal(0, 0.3, r.shape)
        y, S = o.prefill_c2(r, k, v, om, up, S0)
        w = np.exp(-np.exp(om))
        kn = k * (1.0 - w)                       # the normalised key of each token
        ye, Se = brute_force_explicit(r, kn, v, om, np.zeros((H, D)), S0)
        ok &= _close(y, ye + up) and _close(S, Se)
    return ok


def pin_c2_normalised_rows(o):
    g = _rng(13)
    B, T, H, D = 1, 40, 2, 16
    r = g.normal(0, 0.3, (B, T, H, D))
    om = g.uniform(-8.0, 3.0, (B, T, H, D))
    ones = np.ones((B, T, H, D))
    up = g.normal(0, 0.3, (B, T, H, D))
    S0 = np.ones((B, H, D, D))
    y, S = o.prefill_c2(r, ones, ones, om, up, S0)
    y_ref = r.sum(axis=-1, keepdims=True) + up
    return _close(S, np.ones_like(S), 1e-13) and _close(y, y_ref, 1e-12)


def pin_c2_second_value(o):
    r, k, v, om, _, S0 = _inputs(14, 2, 20, 2, 8)
    up = _rng(15).normal(0, 1.0, r.shape)
    y0, S0_ = o.prefill_c2(r, k, v, om, np.zeros_like(r), S0)
    y1, S1_ = o.prefill_c2(r, k, v, om, up, S0)
    return _close(y1 - y0, up) and np.array_equal(S0_, S1_)


def pin_c2_decode(o):
    g = _rng(16)
    B, H, D = 3, 2, 64
    r, k, v, up = (g.normal(0, 0.3, (B, H, D)) for _ in range(4))
    om = g.uniform(-6, 2, (B, H, D))
    S0 = g.normal(0, 0.1, (B, H, D, D))
    y, S = o.decode_step_c2(r, k, v, om, up, S0)
    w = np.exp(-np.exp(om))
    y_ref = np.einsum("bhi,bhij->bhj", r, S0) + up
    S_ref = w[..., None] * S0 + (k * (1.0 - w))[..., :, None] * v[..., None, :]
    return _close(y, y_ref) and _close(S, S_ref)


def pin_gn_moments(o):
    g = _rng(21)
    x = g.normal(0.4, 2.0, (5, 3, 64))
    y = o.groupnorm_gate(x, None, None, 1e-5)
    var = x.var(axis=-1, keepdims=True)
    ok = float(np.max(np.abs(y.mean(axis=-1)))) <= 1e-13   # absolute: the reference is 0
    return ok and _close(y.var(axis=-1, keepdims=True), var / (var + 1e-5), 1e-10)


def pin_gn_torch(o):
    g = _rng(22)
    N, H, D = 7, 4, 64
    x = g.normal(0, 1.0, (N, H, D))
    gam = 1 + 0.1 * g.normal(size=H * D)
    bet = 0.1 * g.normal(size=H * D)
    y = o.groupnorm_gate(x, gam, bet, 1e-5)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x.reshape(N, H * D)), H,
                                         torch.from_numpy(gam), torch.from_numpy(bet), 1e-5)
    return _close(y.reshape(N, H * D), ref.numpy(), 1e-12)


def pin_gn_gate(o):
    g = _rng(23)
    x = g.normal(0, 1.0, (4, 2, 64))
    gam = 1 + 0.1 * g.normal(size=128)
    bet = 0.1 * g.normal(size=128)
    gate = g.normal(0, 1.0, x.shape)
    base = o.groupnorm_gate(x, gam, bet, 1e-5)
    ok = _close(o.groupnorm_gate(x, gam, bet, 1e-5, np.ones_like(x)), base)
    ok &= _close(o.groupnorm_gate(x, gam, bet, 1e-5, 2.0 * np.ones_like(x)), 2.0 * base)
    return ok and _close(o.groupnorm_gate(x, gam, bet, 1e-5, gate), base * gate)


def pin_gn_head_local(o):
    g = _rng(24)
    x = g.normal(0, 1.0, (3, 4, 64))
    x2 = x.copy()
    x2[:, 2] = g.normal(5.0, 3.0, (3, 64))
    a, b = o.groupnorm_gate(x, None, None, 1e-5), o.groupnorm_gate(x2, None, None, 1e-5)
    return np.array_equal(a[:, [0, 1, 3]], b[:, [0, 1, 3]]) and not np.allclose(a[:, 2], b[:, 2])


def _bwd_inputs(seed, B, T, H, D):
    r, k, v, om, u, S0 = _inputs(seed, B, T, H, D, omega=(-3.0, 1.0))
    g = _rng(seed + 100)
    return r, k, v, om, u, S0, g.normal(0, 1.0, r.shape), g.normal(0, 1.0, S0.shape)


def pin_bwd_finite_diff(o):
    r, k, v, om, u, S0, dy, dS = _bwd_inputs(30, 2, 4, 2, 3)
    got = o.backward(r, k, v, om, u, S0, dy, dS)

    def loss(*a):
        y, S = o.prefill(*a)
        return float(np.sum(y * dy) + np.sum(S * dS))

    base = [r, k, v, om, u, S0]
    h = 1e-6
    ok = True
    for idx in range(6):          # got: dr, dk, dv, domega, du, dS0 -- the order of base
        x = base[idx]
        num = np.zeros_like(x)
        for e in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[e] += h
            xm[e] -= h
            ap, am = list(base), list(base)
            ap[idx], am[idx] = xp, xm
            num[e] = (loss(*ap) - loss(*am)) / (2 * h)
        ok &= _close(got[idx], num, rtol=1e-6)
    return ok


def _torch_explicit(r, k, v, om, u, S0):
    """y and final state, explicit-sum form in torch (differentiable), products one by one."""
    B, T, H, D = r.shape
    w = torch.exp(-torch.exp(om))
    ys, finals = [], []
    for b in range(B):
        yb, fb = [], []
        for h in range(H):
            rows = []
            for t in range(T + 1):
                wkv = S0[b, h]
                for j in range(t):
                    wkv = w[b, j, h][:, None] * wkv     # S0 decayed by every earlier token
                for i in range(t):
                    dec = torch.ones(D, dtype=r.dtype)
                    for j in range(i + 1, t):
                        dec = dec * w[b, j, h]
                    wkv = wkv + (dec * k[b, i, h])[:, None] * v[b, i, h][None, :]
                if t < T:
                    rt = r[b, t, h]
                    rows.append(rt @ wkv + torch.sum(rt * u[h] * k[b, t, h]) * v[b, t, h])
                else:
                    fb.append(wkv)
            yb.append(torch.stack(rows))
        ys.append(torch.stack(yb, dim=1))
        finals.append(torch.stack(fb))
    return torch.stack(ys), torch.stack(finals)


def pin_bwd_autograd(o):
    ok = True
    for seed, (B, T, H, D) in [(31, (1, 5, 2, 4)), (32, (2, 3, 1, 6))]:
        r, k, v, om, u, S0, dy, dS = _bwd_inputs(seed, B, T, H, D)
        ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (r, k, v, om, u, S0)]
        y, S = _torch_explicit(*ts)
        (torch.sum(y * torch.tensor(dy)) + torch.sum(S * torch.tensor(dS))).backward()
        got = o.backward(r, k, v, om, u, S0, dy, dS)
        for g_or, t in zip(got, ts):
            ok &= _close(g_or, t.grad.numpy(), rtol=1e-10)
    return ok


def pin_bwd_decay_identity(o):
    r, k, v, om, u, S0, dy, dS = _bwd_inputs(33, 2, 7, 2, 5)
    dr, dk, dv, dom, du, dS0 = o.backward(r, k, v, om, u, S0, dy, dS)
    _, S_T = o.prefill(r, k, v, om, u, S0)
    vdy = np.sum(v * dy, axis=-1, keepdims=True)
    bonus = r * u[None, None] * k * vdy                  # r_t u k_t (v_t . dy_t), per channel
    P = r * dr - bonus                                   # r_s dr_s without the bonus part
    Q = k * dk - bonus                                   # k_s dk_s without the bonus part
    E = np.einsum("bhij,bhij->bhi", S_T, dS)             # <S_T, dS_T> per row
    T = r.shape[1]
    dlog = np.empty_like(r)
    for t in range(T):
        dlog[:, t] = E + P[:, t + 1:].sum(axis=1) - Q[:, t:].sum(axis=1)
    return _close(dom, dlog * (-np.exp(om)), rtol=1e-11)


def pin_c2_bwd_finite_diff(o):
    r, k, v, om, _, S0, dy, dS = _bwd_inputs(35, 2, 4, 1, 3)
    up = _rng(36).normal(0, 0.5, r.shape)
    got = o.backward_c2(r, k, v, om, S0, dy, dS)

    def loss(*a):
        y, S = o.prefill_c2(*a)
        return float(np.sum(y * dy) + np.sum(S * dS))

    base = [r, k, v, om, up, S0]       # got: dr, dk, dv, domega, du', dS0 -- this order
    h = 1e-6
    ok = True
    for idx in range(6):
        x = base[idx]
        num = np.zeros_like(x)
        for e in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[e] += h
            xm[e] -= h
            ap, am = list(base), list(base)
            ap[idx], am[idx] = xp, xm
            num[e] = (loss(*ap) - loss(*am)) / (2 * h)
        ok &= _close(got[idx], num, rtol=1e-6)
    return ok


def _torch_c2_explicit(r, k, v, om, up, S0):
    """Finch-C2: y_t = r_t . sum_{s<t} diag(prod w) (k_s (1 - w_s))^T v_s + decayed S0, plus
    u'_t; final state likewise; products formed one by one (torch, differentiable)."""
    B, T, H, D = r.shape
    w = torch.exp(-torch.exp(om))
    ys, finals = [], []
    for b in range(B):
        yb, fb = [], []
        for h in range(H):
            rows = []
            for t in range(T + 1):
                wkv = S0[b, h]
                for j in range(t):
                    wkv = w[b, j, h][:, None] * wkv
                for i in range(t):
                    dec = torch.ones(D, dtype=r.dtype)
                    for j in range(i + 1, t):
                        dec = dec * w[b, j, h]
                    kn = k[b, i, h] * (1.0 - w[b, i, h])
                    wkv = wkv + (dec * kn)[:, None] * v[b, i, h][None, :]
                if t < T:
                    rows.append(r[b, t, h] @ wkv + up[b, t, h])
                else:
                    fb.append(wkv)
            yb.append(torch.stack(rows))
        ys.append(torch.stack(yb, dim=1))
        finals.append(torch.stack(fb))
    return torch.stack(ys), torch.stack(finals)


def pin_c2_bwd_autograd(o):
    ok = True
    for seed, (B, T, H, D) in [(37, (1, 5, 2, 4)), (38, (2, 3, 1, 5))]:
        r, k, v, om, _, S0, dy, dS = _bwd_inputs(seed, B, T, H, D)
        up = _rng(seed + 1).normal(0, 0.5, r.shape)
        ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True)
              for a in (r, k, v, om, up, S0)]
        y, S = _torch_c2_explicit(*ts)
        (torch.sum(y * torch.tensor(dy)) + torch.sum(S * torch.tensor(dS))).backward()
        got = o.backward_c2(r, k, v, om, S0, dy, dS)
        for g_or, t in zip(got, ts):
            ok &= _close(g_or, t.grad.numpy(), rtol=1e-10)
    return ok


def pin_c2_bwd_decay_identity(o):
    r, k, v, om, _, S0, dy, dS = _bwd_inputs(39, 2, 6, 2, 4)
    up = _rng(40).normal(0, 0.5, r.shape)
    dr, dk, dv, dom, dup, dS0 = o.backward_c2(r, k, v, om, S0, dy, dS)
    _, S_T = o.prefill_c2(r, k, v, om, up, S0)
    w = np.exp(-np.exp(om))
    dkn = dk / (1.0 - w)                 # omega in (-3, 1): 1 - w >= 0.049
    P = r * dr
    Q = k * (1.0 - w) * dkn
    E = np.einsum("bhij,bhij->bhi", S_T, dS)
    T = r.shape[1]
    want = np.empty_like(r)
    for t in range(T):
        dlog = E + P[:, t + 1:].sum(axis=1) - Q[:, t:].sum(axis=1)
        want[:, t] = -np.exp(om[:, t]) * (dlog - dkn[:, t] * k[:, t] * w[:, t])
    return _close(dom, want, rtol=1e-10) and np.array_equal(dup, dy)


def pin_bwd_empty(o):
    r, k, v, om, u, S0, dy, dS = _bwd_inputs(34, 2, 0, 3, 4)
    dr, dk, dv, dom, du, dS0 = o.backward(r, k, v, om, u, S0, dy, dS)
    return np.array_equal(dS0, dS) and not np.any(du) and dr.size == 0


def _gold_inputs(seed, N=7, D=48, Dc=8):
    g = _rng(seed)
    return (g.normal(0, 1.0, (N, D)), g.normal(0, 1.0, (N, Dc)), g.normal(0, 0.2, (Dc, D)),
            g.normal(0, 0.2, (D, D + Dc)), g.normal(1.0, 0.3, D))


def pin_gold_compress_matmul(o):
    x, _, w_kd, _, _ = _gold_inputs(40)
    return _close(o.gold_compress(x, w_kd), x @ w_kd.T, rtol=1e-12)


def pin_gold_decompress_blocks(o):
    x0, c, _, w_ku, gam = _gold_inputs(41)
    D = x0.shape[1]
    z = x0 @ w_ku[:, :D].T + c @ w_ku[:, D:].T
    want = z / np.sqrt(np.mean(z * z, axis=1, keepdims=True) + 1e-3) * gam
    return _close(o.gold_decompress(x0, c, w_ku, gam, 1e-3), want, rtol=1e-12)


def pin_gold_rmsnorm_torch(o):
    x0, c, _, w_ku, gam = _gold_inputs(42)
    x0, c = 0.3 * x0, 0.3 * c          # row mean squares near 0.2, so eps = 0.5 matters
    z = torch.cat([torch.tensor(x0), torch.tensor(c)], dim=1) @ torch.tensor(w_ku).T
    want = torch.nn.functional.rms_norm(z, (z.shape[1],), weight=torch.tensor(gam), eps=0.5)
    return _close(o.gold_decompress(x0, c, w_ku, gam, 0.5), want.numpy(), rtol=1e-12)


def pin_gold_scale_invariance(o):
    x0, c, _, w_ku, gam = _gold_inputs(43)
    a = o.gold_decompress(x0, c, w_ku, gam, 0.0)
    b = o.gold_decompress(7.5 * x0, 7.5 * c, w_ku, gam, 0.0)
    ms = np.mean((a / gam) ** 2, axis=1)
    return _close(a, b, rtol=1e-12) and bool(np.all(np.abs(ms - 1.0) < 1e-12))


PINS = {
    "explicit_sum": pin_explicit_sum,
    "t1_closed_form": pin_t1_closed_form,
    "decode_closed_form": pin_decode_closed_form,
    "linear_attention": pin_linear_attention,
    "zero_decay": pin_zero_decay,
    "geometric": pin_geometric,
    "split_carry": pin_split_carry,
    "linearity": pin_linearity,
    "ln_moments": pin_ln_moments,
    "ln_torch": pin_ln_torch,
    "ln_shift": pin_ln_shift,
    "c2_explicit_sum": pin_c2_explicit_sum,
    "c2_normalised_rows": pin_c2_normalised_rows,
    "c2_second_value": pin_c2_second_value,
    "c2_decode": pin_c2_decode,
    "gn_moments": pin_gn_moments,
    "gn_torch": pin_gn_torch,
    "gn_gate": pin_gn_gate,
    "gn_head_local": pin_gn_head_local,
    "bwd_finite_diff": pin_bwd_finite_diff,
    "bwd_autograd": pin_bwd_autograd,
    "bwd_decay_identity": pin_bwd_decay_identity,
    "bwd_empty": pin_bwd_empty,
    "c2_bwd_finite_diff": pin_c2_bwd_finite_diff,
    "c2_bwd_autograd": pin_c2_bwd_autograd,
    "c2_bwd_decay_identity": pin_c2_bwd_decay_identity,
    "gold_compress_matmul": pin_gold_compress_matmul,
    "gold_decompress_blocks": pin_gold_decompress_blocks,
    "gold_rmsnorm_torch": pin_gold_rmsnorm_torch,
    "gold_scale_invariance": pin_gold_scale_invariance,
}


def run_all(o):
    """Names of the pins that the given oracle fails."""
    failed = []
    for name, fn in PINS.items():
        try:
            ok = bool(fn(o))
        except Exception:  # a crash counts as a failure
            ok = False
        if not ok:
            failed.append(name)
    return failed
