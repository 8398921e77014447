"""Helpers shared by the GPU parity tests: moving inputs to the oracle and the metric.

The parity metric is the one the tolerances are stated in: max|gpu - oracle| divided by
max|oracle| over the compared tensor, taken separately for y and for the final state.
Tolerances: 1e-4 for fp32 I/O, 5e-3 for bf16 I/O.
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 5e-3}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a device or host tensor (bf16 and fp32 convert exactly)."""
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(gpu, ref) -> float:
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    assert np.all(np.isfinite(g)), "non-finite value in GPU output"
    denom = float(np.max(np.abs(r)))
    return float(np.max(np.abs(g - r))) / (denom if denom > 0 else 1.0)


def head_slice(x: torch.Tensor, b, h):
    """[B,T,H,D] -> [1,T,1,D] fp64 copy of one (b,h)."""
    return f64(x[b:b + 1, :, h:h + 1, :])


def oracle_heads(oracle, inp, heads, T=None):
    """Run the oracle on the listed (b,h) heads; returns {(b,h): (y [T,D], S [D,D])}."""
    out = {}
    T = inp["r"].shape[1] if T is None else T
    for (b, h) in heads:
        args = [head_slice(inp[n][:, :T], b, h) for n in ("r", "k", "v", "omega")]
        u = f64(inp["u"][h:h + 1])
        s0 = f64(inp["state0"][b:b + 1, h:h + 1]) if inp.get("state0") is not None else None
        y, S = oracle.prefill(*args, u, s0)
        out[(b, h)] = (y[0, :, 0, :], S[0, 0])
    return out
