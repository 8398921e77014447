"""GPU parity of Finch-C2's backward pass (wkv6c2_backward) against the fp64 oracle's
adjoint: every gradient (dr, dk, dv, domega, du', dS0) element by element, for fp32 and
bf16 I/O, ragged tiles, strong decays, with and without the initial state and final-state
gradient, and the 1.5B-layer shape on sampled heads.  With bf16 I/O dr and dk run on the
tensor cores (a (b,h) whose decays the one-sided factors cannot take falls back to the
scans: covered by a case that mixes both)."""
import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("dr", "dk", "dv", "domega", "duprime", "dS0")


def _problem(seed, B, T, H, dtype, cfg=1, s0=True, ds=True):
    inp = W.make_prefill_inputs(W.CONFIGS[cfg].with_(seed=seed, H=H), DEV, B=B, T=T)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n].float().to(dtype).contiguous()
    g = torch.Generator(device=DEV).manual_seed(seed + 13)
    inp["dy"] = torch.randn((B, T, H, 64), generator=g, device=DEV).to(dtype)
    inp["dS"] = torch.randn((B, H, 64, 64), generator=g, device=DEV) * 0.1 if ds else None
    if not s0:
        inp["state0"] = None
    return inp


def _gpu(inp):
    out = gw.wkv6c2_backward(inp["r"], inp["k"], inp["v"], inp["omega"], inp["state0"],
                             inp["dy"], inp["dS"])
    torch.cuda.synchronize()
    return out


def _oracle(oracle, inp):
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega")]
    s0 = None if inp["state0"] is None else f64(inp["state0"])
    ds = None if inp["dS"] is None else f64(inp["dS"])
    return oracle.backward_c2(*a, s0, f64(inp["dy"]), ds)


def _compare(got, want, tol):
    for name, g, o in zip(NAMES, got, want):
        err = rel_err(g, o)
        assert err <= tol, f"{name}: {err:.3e} > {tol}"


@pytest.mark.parametrize("T", [1, 33, 200])
def test_c2_backward_fp32(oracle, T):
    inp = _problem(10100 + T, B=2, T=T, H=3, dtype=torch.float32, cfg=0)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.float32])


@pytest.mark.parametrize("T", [64, 513])
def test_c2_backward_bf16(oracle, T):
    inp = _problem(10150 + T, B=2, T=T, H=4, dtype=torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_c2_backward_strong_decay_no_state(oracle):
    inp = _problem(10170, B=2, T=150, H=2, dtype=torch.float32, cfg=0, s0=False, ds=False)
    g = torch.Generator(device=DEV).manual_seed(10171)
    inp["omega"] = -9.0 + 13.0 * torch.rand(inp["omega"].shape, generator=g, device=DEV)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.float32])


@pytest.mark.parametrize("T", [1, 65, 130])
def test_c2_backward_bf16_ragged(oracle, T):
    inp = _problem(10160 + T, B=2, T=T, H=3, dtype=torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_c2_backward_bf16_no_state(oracle):
    inp = _problem(10175, B=2, T=200, H=2, dtype=torch.bfloat16, s0=False, ds=False)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_c2_backward_bf16_some_heads_fall_back(oracle):
    """bf16 dr and dk run on the tensor cores per (b,h); one batch row's head with decays
    near zero is redone by the CUDA-core scans, the rest are not."""
    inp = _problem(10176, B=3, T=300, H=3, dtype=torch.bfloat16)
    om = inp["omega"].float()
    om[1, 100:180, 2, ::2] = 3.0
    inp["omega"] = om.to(torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


@pytest.mark.parametrize("segments", [None, "3"])
def test_c2_backward_bf16_extreme_decay_and_split(oracle, monkeypatch, segments):
    """bf16: dv runs through the chunked prefill's query-(1 - w) variant on time-reversed
    copies; decays near zero make it hand sequences to the level kernel, and a forced 3-way
    sequence split runs the segment pre-pass on the reversed sequence."""
    if segments:
        monkeypatch.setenv("GOLDWKV_SEGMENTS", segments)
    inp = _problem(10177, B=2, T=1100, H=2, dtype=torch.bfloat16)
    om = inp["omega"].float()
    om[:, 300:420, 1, ::3] = 3.5
    inp["omega"] = om.to(torch.bfloat16)
    _compare(_gpu(inp), _oracle(oracle, inp), TOL[torch.bfloat16])


def test_c2_backward_duprime_is_dy():
    inp = _problem(10180, B=1, T=70, H=2, dtype=torch.bfloat16)
    out = _gpu(inp)
    assert torch.equal(out[4], inp["dy"])


def test_c2_backward_1p5b_layer_sampled_heads(oracle):
    cfg = W.CONFIGS[1]
    inp = _problem(cfg.seed + 3, B=cfg.B, T=cfg.T, H=cfg.H, dtype=torch.bfloat16)
    got = _gpu(inp)
    for b, h in ((0, 4), (6, 29)):
        sub = {n: inp[n][b:b + 1, :, h:h + 1].contiguous() for n in ("r", "k", "v", "omega", "dy")}
        sub["state0"] = inp["state0"][b:b + 1, h:h + 1].contiguous()
        sub["dS"] = inp["dS"][b:b + 1, h:h + 1].contiguous()
        want = _oracle(oracle, sub)
        for name, g, o in zip(NAMES, got, want):
            gs = g[b:b + 1, h:h + 1] if name == "dS0" else g[b:b + 1, :, h:h + 1]
            err = rel_err(gs, o)
            assert err <= TOL[torch.bfloat16], f"{name} head ({b},{h}): {err:.3e}"
