"""Seeded synthetic workloads for the WKV6 prefill / decode path.

This module only draws random inputs; it holds none of the recurrence's arithmetic, so
both the CUDA path's tests and the fp64 oracle can take their inputs from it.

Shapes follow the GoldFinch workloads: a 1.5B-class layer (d_model 2048 = 32 heads x 64),
a 4096-wide long-context layer, a batched decode step and a decay-extreme case with the
full-width LayerNorm of Finch-C2.  Distributions (``N(0, s)`` read as standard deviation
``s``):

* r, k, v ~ N(0, 1) / 8, drawn in fp32 and rounded to the I/O dtype;
* omega (the decay logit d_t, so that w = exp(-exp(omega))) ~ U(lo, hi), or, in the
  decay-extreme case, each (head, channel) is assigned once to a "slow" class
  (omega ~ U(-12, -6), w ~ 1) or a "fast" class (omega ~ U(2, 4), w ~ 0), half each;
* u ~ N(0, 0.5) per head x channel, fp32;
* initial state zero, or ~ N(0, 0.1) fp32;
* LayerNorm gamma ~ 1 + N(0, 0.1), beta ~ N(0, 0.1) over d_model, eps 1e-5.

Large tensors are drawn in blocks of ``GEN_BLOCK_TOKENS`` tokens so that the fp32
temporaries stay small; the block size is part of the recipe (same seed, same values).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

GEN_BLOCK_TOKENS = 4096


@dataclass(frozen=True)
class WkvConfig:
    name: str
    B: int
    T: int
    H: int
    D: int = 64
    io: str = "bf16"              # "f32" or "bf16"
    omega: tuple = (-6.0, 1.0)    # (lo, hi) of U(lo, hi), or "extreme"
    state0: str = "zero"          # "zero" or "normal0.1"
    ln: bool = False
    steps: int = 0                # decode steps (0: prefill workload)
    seed: int = 0

    @property
    def dtype(self) -> torch.dtype:
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def with_(self, **kw) -> "WkvConfig":
        return replace(self, **kw)


CONFIGS = [
    WkvConfig("wkv6_tiny_f32", B=1, T=64, H=2, io="f32", seed=1000),
    WkvConfig("wkv6_prefill_1p5b_layer", B=8, T=4096, H=32, state0="normal0.1", seed=1001),
    WkvConfig("wkv6_prefill_long_ctx", B=1, T=262144, H=64, omega=(-8.0, 0.0), seed=1002),
    WkvConfig("wkv6_decode_step", B=256, T=1, H=32, state0="normal0.1", steps=100, seed=1003),
    WkvConfig("wkv6_decay_extreme_ln", B=4, T=16384, H=32, omega="extreme", ln=True, seed=1004),
]
BY_NAME = {c.name: c for c in CONFIGS}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_tokens(g, shape, std, dtype, device):
    """N(0, std) over [B, T, ...], drawn per token block in fp32 then rounded."""
    B, T = shape[0], shape[1]
    out = torch.empty(shape, dtype=dtype, device=device)
    for t0 in range(0, T, GEN_BLOCK_TOKENS):
        t1 = min(T, t0 + GEN_BLOCK_TOKENS)
        blk = torch.randn((B, t1 - t0) + tuple(shape[2:]), generator=g, device=device,
                          dtype=torch.float32)
        out[:, t0:t1] = (blk * std).to(dtype)
    return out


def _uniform_tokens(g, shape, lo, hi, dtype, device):
    B, T = shape[0], shape[1]
    out = torch.empty(shape, dtype=dtype, device=device)
    for t0 in range(0, T, GEN_BLOCK_TOKENS):
        t1 = min(T, t0 + GEN_BLOCK_TOKENS)
        blk = torch.rand((B, t1 - t0) + tuple(shape[2:]), generator=g, device=device,
                         dtype=torch.float32)
        out[:, t0:t1] = (lo + (hi - lo) * blk).to(dtype)
    return out


def _extreme_omega(g, shape, dtype, device):
    """Half of the (head, channel) pairs slow (U(-12,-6)), half fast (U(2,4))."""
    B, T, H, D = shape
    perm = torch.randperm(H * D, generator=g, device=device)
    slow = torch.zeros(H * D, dtype=torch.bool, device=device)
    slow[perm[: (H * D) // 2]] = True
    slow = slow.view(H, D)
    lo = torch.where(slow, torch.tensor(-12.0, device=device), torch.tensor(2.0, device=device))
    hi = torch.where(slow, torch.tensor(-6.0, device=device), torch.tensor(4.0, device=device))
    out = torch.empty(shape, dtype=dtype, device=device)
    for t0 in range(0, T, GEN_BLOCK_TOKENS):
        t1 = min(T, t0 + GEN_BLOCK_TOKENS)
        blk = torch.rand((B, t1 - t0, H, D), generator=g, device=device, dtype=torch.float32)
        out[:, t0:t1] = (lo + (hi - lo) * blk).to(dtype)
    return out, slow


def make_prefill_inputs(cfg: WkvConfig, device="cpu", *, B=None, T=None, seed=None):
    """Seeded prefill inputs; B/T may be overridden (same distributions, smaller case)."""
    B = cfg.B if B is None else B
    T = cfg.T if T is None else T
    H, D, dt = cfg.H, cfg.D, cfg.dtype
    g = _gen(cfg.seed if seed is None else seed, device)
    shape = (B, T, H, D)
    r = _normal_tokens(g, shape, 0.125, dt, device)
    k = _normal_tokens(g, shape, 0.125, dt, device)
    v = _normal_tokens(g, shape, 0.125, dt, device)
    slow = None
    if cfg.omega == "extreme":
        omega, slow = _extreme_omega(g, shape, dt, device)
    else:
        omega = _uniform_tokens(g, shape, cfg.omega[0], cfg.omega[1], dt, device)
    u = torch.randn((H, D), generator=g, device=device, dtype=torch.float32) * 0.5
    if cfg.state0 == "zero":
        state0 = torch.zeros((B, H, D, D), dtype=torch.float32, device=device)
    else:
        state0 = torch.randn((B, H, D, D), generator=g, device=device, dtype=torch.float32) * 0.1
    out = dict(r=r, k=k, v=v, omega=omega, u=u, state0=state0, slow=slow)
    if cfg.ln:
        out["gamma"] = 1.0 + 0.1 * torch.randn((H * D,), generator=g, device=device,
                                               dtype=torch.float32)
        out["beta"] = 0.1 * torch.randn((H * D,), generator=g, device=device, dtype=torch.float32)
        out["eps"] = 1e-5
    return out


def _share_params(out, base):
    for n in ("u", "gamma", "beta"):
        if n in base:
            out[n] = base[n]
    return out


def make_prefill_shard(cfg: WkvConfig, device, rank: int, **kw):
    """Rank `rank`'s batch in a data-parallel run: its own tokens and initial state (seed
    cfg.seed + 17 * rank), the layer's parameters u (and LayerNorm gamma, beta) those of
    rank 0, as every rank holds the same layer."""
    out = make_prefill_inputs(cfg, device, seed=cfg.seed + 17 * rank, **kw)
    return _share_params(out, make_prefill_inputs(cfg, device, **kw)) if rank else out


def make_decode_shard(cfg: WkvConfig, device, rank: int, **kw):
    """As make_prefill_shard, for the decode inputs."""
    out = make_decode_inputs(cfg, device, seed=cfg.seed + 17 * rank, **kw)
    return _share_params(out, make_decode_inputs(cfg, device, **kw)) if rank else out


def make_decode_inputs(cfg: WkvConfig, device="cpu", *, B=None, steps=None, seed=None):
    """Seeded decode inputs: per-step r,k,v,omega [steps, B, H, D], u, initial state."""
    B = cfg.B if B is None else B
    steps = (cfg.steps or 1) if steps is None else steps
    H, D, dt = cfg.H, cfg.D, cfg.dtype
    g = _gen(cfg.seed if seed is None else seed, device)
    shape = (steps, B, H, D)

    def normal():
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * 0.125).to(dt)

    r, k, v = normal(), normal(), normal()
    lo, hi = cfg.omega
    omega = (lo + (hi - lo) * torch.rand(shape, generator=g, device=device,
                                         dtype=torch.float32)).to(dt)
    u = torch.randn((H, D), generator=g, device=device, dtype=torch.float32) * 0.5
    if cfg.state0 == "zero":
        state0 = torch.zeros((B, H, D, D), dtype=torch.float32, device=device)
    else:
        state0 = torch.randn((B, H, D, D), generator=g, device=device, dtype=torch.float32) * 0.1
    return dict(r=r, k=k, v=v, omega=omega, u=u, state0=state0)
