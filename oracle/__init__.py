"""TEST INFRASTRUCTURE ONLY: fp64 CPU oracle for the Finch-C2 / RWKV-6 WKV recurrence.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product library (libgoldwkv) never
links, loads or calls it, and the two share no code.

The arithmetic lives in ``wkv6_oracle.c`` (plain sequential loops, fp64), which follows
the GoldFinch review page, section 3.4 "Finch-C2 Time Mixing": decay
``w_t = exp(-exp(d_t))`` ("Data-dependent decay"), the state sum
``wkv_t = sum_{i<t} diag(prod_{j=i+1}^{t-1} w_j) k_i^T v_i`` ("Recurrent state update and
output"), readout ``r_t . wkv_t`` plus the base-Finch static bonus ``r_t . diag(u) k_t^T v_t``,
and LayerNorm over the concatenated heads; base Finch's per-head GroupNorm and gate; the
backward pass of the base recurrence; GOLD key compression and TokenCat decompression
(section 3.4 "GOLD Key Compression and TokenCat Decompression").  This module only
builds/loads the shared object and marshals numpy arrays.

Pins: every entry point is checked by ``tests/test_oracle_pins.py`` against brute-force
sums, closed forms and invariants that do not call this code (see that file's header).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "wkv6_oracle.c"
_BUILD = _HERE / "_build"
_SO = _BUILD / "libwkv6_oracle.so"


def build(src: Path = _SRC, out: Path = _SO, extra_flags=()) -> Path:
    """Compile the oracle C source with gcc into a shared object (no -march tuning)."""
    out.parent.mkdir(parents=True, exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", *extra_flags,
           str(src), "-o", str(out), "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(so: Path, src: Path) -> bool:
    return (not so.exists()) or so.stat().st_mtime < src.stat().st_mtime


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


class Oracle:
    """ctypes front end of one compiled oracle shared object."""

    def __init__(self, so_path: Path | str | None = None):
        if so_path is None:
            if _needs_build(_SO, _SRC):
                build()
            so_path = _SO
        self.path = Path(so_path)
        lib = ctypes.CDLL(str(self.path))
        dp = ctypes.POINTER(ctypes.c_double)
        lib.wkv6_oracle_prefill.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.wkv6_oracle_prefill.restype = ctypes.c_int
        lib.wkv6_oracle_decode_step.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.wkv6_oracle_decode_step.restype = ctypes.c_int
        lib.wkv6c2_oracle_prefill.argtypes = lib.wkv6_oracle_prefill.argtypes
        lib.wkv6c2_oracle_prefill.restype = ctypes.c_int
        lib.wkv6c2_oracle_decode_step.argtypes = lib.wkv6_oracle_decode_step.argtypes
        lib.wkv6c2_oracle_decode_step.restype = ctypes.c_int
        lib.wkv6_oracle_layernorm.argtypes = [ctypes.c_long, ctypes.c_int, dp, dp, dp,
                                              ctypes.c_double, dp]
        lib.wkv6_oracle_layernorm.restype = ctypes.c_int
        lib.wkv6_oracle_groupnorm_gate.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, dp, dp,
                                                   dp, ctypes.c_double, dp, dp]
        lib.wkv6_oracle_groupnorm_gate.restype = ctypes.c_int
        lib.wkv6_oracle_backward.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                             dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp]
        lib.wkv6_oracle_backward.restype = ctypes.c_int
        lib.wkv6c2_oracle_backward.argtypes = [ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                               ctypes.c_int] + [dp] * 13
        lib.wkv6c2_oracle_backward.restype = ctypes.c_int
        lib.gold_oracle_compress.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, dp, dp, dp]
        lib.gold_oracle_compress.restype = ctypes.c_int
        lib.gold_oracle_decompress.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, dp, dp, dp,
                                               dp, ctypes.c_double, dp]
        lib.gold_oracle_decompress.restype = ctypes.c_int
        self._lib = lib

    @staticmethod
    def _f64(a):
        if a is None:
            return None
        return np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    @staticmethod
    def _ptr(a):
        if a is None:
            return None
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))

    def prefill(self, r, k, v, omega, u, state_in=None, nthreads: int | None = None):
        """r,k,v,omega: [B,T,H,D]; u: [H,D]; state_in: [B,H,D,D] or None.

        Returns (y [B,T,H,D], state_out [B,H,D,D]) as float64 arrays.
        """
        r, k, v, omega, u = (self._f64(x) for x in (r, k, v, omega, u))
        s_in = self._f64(state_in)
        B, T, H, D = r.shape
        assert k.shape == v.shape == omega.shape == r.shape and u.shape == (H, D)
        if s_in is not None:
            assert s_in.shape == (B, H, D, D)
        y = np.empty_like(r)
        s_out = np.empty((B, H, D, D), dtype=np.float64)
        rc = self._lib.wkv6_oracle_prefill(B, T, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                           self._ptr(omega), self._ptr(u), self._ptr(s_in),
                                           self._ptr(y), self._ptr(s_out),
                                           nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle prefill failed rc={rc}")
        return y, s_out

    def decode_step(self, r, k, v, omega, u, state, nthreads: int | None = None):
        """r,k,v,omega: [B,H,D]; state [B,H,D,D] (not modified). Returns (y, new_state)."""
        r, k, v, omega, u = (self._f64(x) for x in (r, k, v, omega, u))
        st = np.array(state, dtype=np.float64, copy=True, order="C")
        B, H, D = r.shape
        y = np.empty_like(r)
        rc = self._lib.wkv6_oracle_decode_step(B, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                               self._ptr(omega), self._ptr(u), self._ptr(st),
                                               self._ptr(y), nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle decode failed rc={rc}")
        return y, st

    def backward(self, r, k, v, omega, u, state_in, dy, dstate_out=None):
        """Gradients of prefill: given dy = dL/dy [B,T,H,D] and dstate_out = dL/dstate_out
        [B,H,D,D] (None: zero), returns (dr, dk, dv, domega [B,T,H,D], du [H,D] summed over
        b and t, dstate_in [B,H,D,D]) as float64 arrays.  state_in None means zeros."""
        r, k, v, omega, u, dy = (self._f64(x) for x in (r, k, v, omega, u, dy))
        s_in, ds_out = self._f64(state_in), self._f64(dstate_out)
        B, T, H, D = r.shape
        assert k.shape == v.shape == omega.shape == dy.shape == r.shape and u.shape == (H, D)
        dr, dk, dv, dom = (np.empty_like(r) for _ in range(4))
        du = np.empty((H, D), dtype=np.float64)
        ds_in = np.empty((B, H, D, D), dtype=np.float64)
        rc = self._lib.wkv6_oracle_backward(B, T, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                            self._ptr(omega), self._ptr(u), self._ptr(s_in),
                                            self._ptr(dy), self._ptr(ds_out), self._ptr(dr),
                                            self._ptr(dk), self._ptr(dv), self._ptr(dom),
                                            self._ptr(du), self._ptr(ds_in))
        if rc != 0:
            raise RuntimeError(f"oracle backward failed rc={rc}")
        return dr, dk, dv, dom, du, ds_in

    def backward_c2(self, r, k, v, omega, state_in, dy, dstate_out=None):
        """Gradients of prefill_c2: (dr, dk, dv, domega, duprime [B,T,H,D], dstate_in
        [B,H,D,D]) for dy [B,T,H,D] and dstate_out [B,H,D,D] (None: zero); fp64."""
        r, k, v, omega, dy = (self._f64(x) for x in (r, k, v, omega, dy))
        s_in, ds_out = self._f64(state_in), self._f64(dstate_out)
        B, T, H, D = r.shape
        assert k.shape == v.shape == omega.shape == dy.shape == r.shape
        dr, dk, dv, dom, dup = (np.empty_like(r) for _ in range(5))
        ds_in = np.empty((B, H, D, D), dtype=np.float64)
        rc = self._lib.wkv6c2_oracle_backward(B, T, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                              self._ptr(omega), self._ptr(s_in), self._ptr(dy),
                                              self._ptr(ds_out), self._ptr(dr), self._ptr(dk),
                                              self._ptr(dv), self._ptr(dom), self._ptr(dup),
                                              self._ptr(ds_in))
        if rc != 0:
            raise RuntimeError(f"oracle backward_c2 failed rc={rc}")
        return dr, dk, dv, dom, dup, ds_in

    def prefill_c2(self, r, k, v, omega, uprime, state_in=None, nthreads: int | None = None):
        """Finch-C2 exact form: key k (1 - w), second value uprime [B,T,H,D] added to the
        readout (no static bonus).  Same shapes and returns as prefill."""
        r, k, v, omega, up = (self._f64(x) for x in (r, k, v, omega, uprime))
        B, T, H, D = r.shape
        s_in = None if state_in is None else self._f64(state_in)
        y = np.empty_like(r)
        s_out = np.empty((B, H, D, D), dtype=np.float64)
        rc = self._lib.wkv6c2_oracle_prefill(B, T, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                             self._ptr(omega), self._ptr(up), self._ptr(s_in),
                                             self._ptr(y), self._ptr(s_out),
                                             nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle C2 prefill failed rc={rc}")
        return y, s_out

    def decode_step_c2(self, r, k, v, omega, uprime, state, nthreads: int | None = None):
        """Finch-C2 step: r,k,v,omega,uprime [B,H,D]; state [B,H,D,D] (not modified)."""
        r, k, v, omega, up = (self._f64(x) for x in (r, k, v, omega, uprime))
        st = np.array(state, dtype=np.float64, copy=True, order="C")
        B, H, D = r.shape
        y = np.empty_like(r)
        rc = self._lib.wkv6c2_oracle_decode_step(B, H, D, self._ptr(r), self._ptr(k), self._ptr(v),
                                                 self._ptr(omega), self._ptr(up), self._ptr(st),
                                                 self._ptr(y), nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle C2 decode failed rc={rc}")
        return y, st

    def prefill_c2_ln(self, r, k, v, omega, uprime, state_in, gamma, beta, eps=1e-5, nthreads=None):
        """Finch-C2 prefill followed by LayerNorm over the concatenated heads."""
        y, s = self.prefill_c2(r, k, v, omega, uprime, state_in, nthreads)
        B, T, H, D = y.shape
        yl = self.layernorm(y.reshape(B, T, H * D), gamma, beta, eps).reshape(B, T, H, D)
        return yl, s, y

    def layernorm(self, x, gamma=None, beta=None, eps: float = 1e-5):
        """LayerNorm over the last axis of x (any leading shape), fp64."""
        x = self._f64(x)
        C = x.shape[-1]
        N = x.size // C
        g = self._f64(gamma)
        b = self._f64(beta)
        out = np.empty_like(x)
        rc = self._lib.wkv6_oracle_layernorm(N, C, self._ptr(x), self._ptr(g), self._ptr(b),
                                             float(eps), self._ptr(out))
        if rc != 0:
            raise RuntimeError(f"oracle layernorm failed rc={rc}")
        return out

    def groupnorm_gate(self, x, gamma=None, beta=None, eps: float = 1e-5, gate=None):
        """Per-head GroupNorm of x [..., H, D] (each head's D channels), affine gamma/beta
        [H*D], then times gate [..., H, D] (or 1), fp64."""
        x = self._f64(x)
        H, D = x.shape[-2], x.shape[-1]
        N = x.size // (H * D)
        g, b, gt = self._f64(gamma), self._f64(beta), self._f64(gate)
        out = np.empty_like(x)
        rc = self._lib.wkv6_oracle_groupnorm_gate(N, H, D, self._ptr(x), self._ptr(g), self._ptr(b),
                                                  float(eps), self._ptr(gt), self._ptr(out))
        if rc != 0:
            raise RuntimeError(f"oracle groupnorm failed rc={rc}")
        return out

    def prefill_gn(self, r, k, v, omega, u, state_in, gamma, beta, eps=1e-5, gate=None, nthreads=None):
        """Base-Finch output: prefill, then per-head GroupNorm and the gate."""
        y, s = self.prefill(r, k, v, omega, u, state_in, nthreads)
        return self.groupnorm_gate(y, gamma, beta, eps, gate), s, y

    def prefill_ln(self, r, k, v, omega, u, state_in, gamma, beta, eps=1e-5, nthreads=None):
        """Prefill followed by LayerNorm over the concatenated heads (H*D) of each token."""
        y, s = self.prefill(r, k, v, omega, u, state_in, nthreads)
        B, T, H, D = y.shape
        yl = self.layernorm(y.reshape(B, T, H * D), gamma, beta, eps).reshape(B, T, H, D)
        return yl, s, y

    def gold_compress(self, x, w_kd):
        """GOLD compression c = x W_KD; x [..., D], w_kd [Dc, D] (rows of the map). fp64."""
        x, w = self._f64(x), self._f64(w_kd)
        D, Dc = x.shape[-1], w.shape[0]
        assert w.shape == (Dc, D)
        xs = np.ascontiguousarray(x.reshape(-1, D))
        c = np.empty((xs.shape[0], Dc))
        rc = self._lib.gold_oracle_compress(xs.shape[0], D, Dc, self._ptr(xs), self._ptr(w),
                                            self._ptr(c))
        if rc != 0:
            raise RuntimeError(f"oracle gold_compress failed rc={rc}")
        return c.reshape(*x.shape[:-1], Dc)

    def gold_decompress(self, x0, c, w_ku, gamma=None, eps: float = 1e-6):
        """TokenCat decompression RMSNorm(concat(x0, c) W_KU); x0 [..., D], c [..., Dc], w_ku
        [D, D + Dc] (rows of the map), gamma [D] or None. fp64."""
        x0, c, w, g = self._f64(x0), self._f64(c), self._f64(w_ku), self._f64(gamma)
        D, Dc = x0.shape[-1], c.shape[-1]
        assert w.shape == (D, D + Dc) and x0.shape[:-1] == c.shape[:-1]
        xs = np.ascontiguousarray(x0.reshape(-1, D))
        cs = np.ascontiguousarray(c.reshape(-1, Dc))
        kd = np.empty_like(xs)
        rc = self._lib.gold_oracle_decompress(xs.shape[0], D, Dc, self._ptr(xs), self._ptr(cs),
                                              self._ptr(w), self._ptr(g), float(eps), self._ptr(kd))
        if rc != 0:
            raise RuntimeError(f"oracle gold_decompress failed rc={rc}")
        return kd.reshape(x0.shape)


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``wkv6_oracle.c`` (compiled on first use if missing or stale)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default

