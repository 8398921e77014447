"""GPU parity of the backward pass (wkv6_backward) against the fp64 oracle's adjoint.

Every gradient (dr, dk, dv, domega, du, dS0) is compared element by element at sizes that
span several 32-token tiles and a ragged tail, for fp32 and bf16 I/O, with and without an
initial state and a final-state gradient; the 1.5B-layer shape (B8 T4096 H32, bf16) is
checked on sampled heads.  With bf16 I/O dv comes from the chunked tensor-core prefill run
on time-reversed copies, and dr from the tensor-core dr kernel (a (b,h) whose decays it
cannot take falls back to the CUDA-core scan): extreme decays (hand-over to the level
kernel, dr fallback) and a forced sequence split cover those paths.  Also: the empty sequence, determinism and argument
checks.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("dr", "dk", "dv", "domega", "du", "dS0")


def _problem(seed, B, T, H, dtype, cfg=1, s0=True, ds=True):
    inp = W.make_prefill_inputs(W.CONFIGS[cfg].with_(seed=seed, H=H), DEV, B=B, T=T)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n].float().to(dtype).contiguous()
    g = torch.Generator(device=DEV).manual_seed(seed + 11)
    inp["dy"] = torch.randn((B, T, H, 64), generator=g, device=DEV).to(dtype)
    inp["dS"] = torch.randn((B, H, 64, 64), generator=g, device=DEV) * 0.1 if ds else None
    if not s0:
        inp["state0"] = None
    return inp


def _gpu(inp):
    out = gw.wkv6_backward(inp["r"], inp["k"], inp["v"], inp["omega"], inp["u"], inp["state0"],
                           inp["dy"], inp["dS"])
    torch.cuda.synchronize()
    return out


def _oracle(oracle, inp):
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega", "u")]
    s0 = None if inp["state0"] is None else f64(inp["state0"])
    ds = None if inp["dS"] is None else f64(inp["dS"])
    return oracle.backward(*a, s0, f64(inp["dy"]), ds)


def _compare(got, want, tol):
    for name, g, o in zip(NAMES, got, want):
        err = rel_err(g, o)
        assert err <= tol, f"{name}: {err:.3e} > {tol}"


@pytest.mark.parametrize("T", [1, 31, 32, 33, 200])
def test_backward_fp32(oracle, T):
    inp = _problem(9800 + T, B=2, T=T, H=3, dtype=torch.float32, cfg=0)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.float32])


@pytest.mark.parametrize("T", [1, 64, 65, 130, 513])
def test_backward_bf16(oracle, T):
    inp = _problem(9850 + T, B=2, T=T, H=4, dtype=torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_backward_bf16_zero_state_no_state_gradient(oracle):
    """The tensor-core dr pass with no initial state and no final-state gradient (E = 0)."""
    inp = _problem(9871, B=3, T=200, H=2, dtype=torch.bfloat16, s0=False, ds=False)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_backward_bf16_some_heads_fall_back(oracle):
    """bf16 dr runs on the tensor cores per (b,h) while every chunk's decay range fits the
    one-sided factorisation; one batch row's head with decays near zero is redone by the
    CUDA-core scan, the rest are not."""
    inp = _problem(9872, B=3, T=300, H=3, dtype=torch.bfloat16)
    om = inp["omega"].float()
    om[1, 100:180, 2, ::2] = 3.0
    inp["omega"] = om.to(torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_backward_zero_state_no_state_gradient(oracle):
    inp = _problem(9870, B=3, T=100, H=2, dtype=torch.float32, cfg=0, s0=False, ds=False)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.float32])


def test_backward_strong_decay(oracle):
    """Decays down to exp(-e^4) and up to nearly 1 in one sequence."""
    inp = _problem(9880, B=2, T=150, H=2, dtype=torch.float32, cfg=0)
    g = torch.Generator(device=DEV).manual_seed(9881)
    inp["omega"] = -9.0 + 13.0 * torch.rand(inp["omega"].shape, generator=g, device=DEV)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.float32])


@pytest.mark.parametrize("segments", [None, "3"])
def test_backward_bf16_extreme_decay_and_split(oracle, monkeypatch, segments):
    """bf16: dv runs through the chunked prefill on time-reversed copies; decays near zero
    make it hand sequences to the level kernel, and a forced 3-way sequence split runs the
    segment pre-pass on the reversed sequence."""
    if segments:
        monkeypatch.setenv("GOLDWKV_SEGMENTS", segments)
    inp = _problem(9895, B=2, T=1100, H=2, dtype=torch.bfloat16)
    om = inp["omega"].float()
    om[:, 300:420, 1, ::3] = 3.5
    inp["omega"] = om.to(torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_backward_empty_sequence():
    inp = _problem(9890, B=2, T=0, H=3, dtype=torch.bfloat16)
    dr, dk, dv, dom, du, ds0 = _gpu(inp)
    assert dr.numel() == 0 and bool((du == 0).all())
    assert torch.equal(ds0, inp["dS"])


def test_backward_deterministic():
    inp = _problem(9900, B=2, T=300, H=4, dtype=torch.bfloat16)
    a, b = _gpu(inp), _gpu(inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_1p5b_layer_sampled_heads(oracle):
    """B8 T4096 H32 bf16 on the GPU; the oracle recomputes every batch row of head 5 (so du
    of that head is complete) and head 27 of row 3."""
    cfg = W.CONFIGS[1]
    inp = _problem(cfg.seed, B=cfg.B, T=cfg.T, H=cfg.H, dtype=torch.bfloat16)
    got = _gpu(inp)
    for bs, h in ((slice(0, cfg.B), 5), (slice(3, 4), 27)):
        sub = {n: inp[n][bs, :, h:h + 1].contiguous() for n in ("r", "k", "v", "omega", "dy")}
        sub["u"] = inp["u"][h:h + 1].contiguous()
        sub["state0"] = inp["state0"][bs, h:h + 1].contiguous()
        sub["dS"] = inp["dS"][bs, h:h + 1].contiguous()
        want = _oracle(oracle, sub)
        for name, g, o in zip(NAMES, got, want):
            if name == "du":
                if bs.stop - bs.start != cfg.B:
                    continue             # du sums over every batch row
                g = g[h:h + 1]
            elif name == "dS0":
                g = g[bs, h:h + 1]
            else:
                g = g[bs, :, h:h + 1]
            err = rel_err(g, o)
            assert err <= TOL[torch.bfloat16], f"{name} head {h}: {err:.3e}"


def test_backward_argument_checks():
    inp = _problem(9910, B=1, T=40, H=2, dtype=torch.float32, cfg=0)
    B, T, H, D = 1, 40, 2, 64
    L = bd.load()
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    outs = [torch.full((B, T, H, D), 3.0, device=DEV) for _ in range(4)]
    du = torch.full((H, D), 3.0, device=DEV)
    ws = torch.empty(bd.backward_workspace_bytes(B, T, H, D, torch.float32), dtype=torch.uint8,
                     device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(dr, ws_t, ws_bytes):
        return L.wkv6_backward(vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]),
                               vp(inp["u"]), vp(inp["state0"]), vp(inp["dy"]), vp(inp["dS"]),
                               vp(dr), vp(outs[1]), vp(outs[2]), vp(outs[3]), vp(du), None,
                               B, T, H, D, bd.WKV_F32, vp(ws_t), ws_bytes, stream)

    assert call(inp["dy"], ws, ws.numel()) == bd.WKV_ERR_INVALID_ARG       # dr on top of dy
    assert call(outs[1], ws, ws.numel()) == bd.WKV_ERR_INVALID_ARG         # dr on top of dk
    assert call(outs[0], ws, ws.numel() - 4) == bd.WKV_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert all(bool((o == 3.0).all()) for o in outs) and bool((du == 3.0).all())
    assert call(outs[0], ws, ws.numel()) == bd.WKV_OK
