"""GPU parity of Finch-C2's exact time mixing (wkv6c2_prefill / wkv6c2_decode_step) against
the fp64 oracle: key normalised by 1 - w, second value u' added to the readout, no static
bonus.  Every kernel path is covered: the fast chunked kernel, the level-factorised kernel
(hand-over and extreme decay from the start), the sequence split, the fp32 recurrence,
LayerNorm, and the decode step.
"""
import ctypes

import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, oracle_heads, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(seed, B, T, H, dtype=torch.bfloat16, cfg=1):
    base = W.CONFIGS[cfg].with_(seed=seed)
    inp = W.make_prefill_inputs(base, DEV, B=B, T=T)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n][:, :, :H].float().to(dtype).contiguous()
    inp["state0"] = inp["state0"][:, :H].contiguous()
    g = torch.Generator(device=DEV).manual_seed(seed + 1)
    inp["uprime"] = (torch.randn(inp["r"].shape, generator=g, device=DEV) * 0.125).to(dtype)
    return inp


def _run(inp, ln=None, state=True):
    a = [inp[n] for n in ("r", "k", "v", "omega", "uprime")]
    y, s = gw.wkv6c2_prefill(*a, inp["state0"] if state else None, ln=ln)
    torch.cuda.synchronize()
    return y, s


def _oracle(oracle, inp, state=True):
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega", "uprime")]
    return oracle.prefill_c2(*a, f64(inp["state0"]) if state else None)


@pytest.mark.parametrize("T", [1, 64, 65, 200, 513])
def test_c2_fast_kernel(oracle, T):
    inp = _problem(8000 + T, B=2, T=T, H=3)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("extreme_from", [0, 130])
def test_c2_level_kernel(oracle, extreme_from):
    """Channels with w ~ 0 from token `extreme_from`: the fast kernel hands the rest of the
    sequence (and its state) to the level kernel, which must apply the same C2 form."""
    inp = _problem(8100 + extreme_from, B=2, T=300, H=3)
    om = inp["omega"].float()
    om[:, extreme_from:, :, ::3] = 3.5
    inp["omega"] = om.to(torch.bfloat16)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_c2_sequence_split(oracle, monkeypatch):
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "3")
    inp = _problem(8200, B=2, T=1100, H=3)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_c2_zero_state_and_normalised_rows(oracle):
    """The page's normalisation property end to end: k = v = 1 and unit state rows stay unit
    rows for any decay, through the tensor-core path."""
    inp = _problem(8300, B=1, T=256, H=2)
    inp["k"] = torch.ones_like(inp["k"])
    inp["v"] = torch.ones_like(inp["v"])
    inp["state0"] = torch.ones_like(inp["state0"])
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert (s - 1.0).abs().max().item() <= TOL[torch.bfloat16]


def test_c2_fp32_recurrence(oracle):
    inp = _problem(8400, B=2, T=150, H=2, dtype=torch.float32, cfg=0)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.float32]
    assert rel_err(s, so) <= TOL[torch.float32]


def test_c2_layernorm(oracle):
    inp = _problem(8500, B=2, T=130, H=4)
    g = torch.Generator(device=DEV).manual_seed(8501)
    gamma = 1.0 + 0.1 * torch.randn(4 * 64, generator=g, device=DEV)
    beta = 0.1 * torch.randn(4 * 64, generator=g, device=DEV)
    y, s = _run(inp, ln=(gamma, beta, 1e-5))
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega", "uprime")]
    yo, so, _ = oracle.prefill_c2_ln(*a, f64(inp["state0"]), f64(gamma), f64(beta), 1e-5)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_c2_decode_steps(oracle, dtype):
    g = torch.Generator(device=DEV).manual_seed(8600)
    B, H, D, steps = 16, 4, 64, 5
    mk = lambda s_: (torch.randn((B, H, D), generator=g, device=DEV) * s_).to(dtype)
    state = torch.randn((B, H, D, D), generator=g, device=DEV) * 0.1
    s_ref = f64(state)
    for _ in range(steps):
        r, k, v, up = mk(0.125), mk(0.125), mk(0.125), mk(0.125)
        om = (-6.0 + 7.0 * torch.rand((B, H, D), generator=g, device=DEV)).to(dtype)
        y = gw.wkv6c2_decode_step(r, k, v, om, up, state)
        torch.cuda.synchronize()
        yo, s_ref = oracle.decode_step_c2(f64(r), f64(k), f64(v), f64(om), f64(up), s_ref)
        assert rel_err(y, yo) <= TOL[dtype]
    assert rel_err(state, s_ref) <= TOL[dtype]


def test_c2_full_layer_shape_sampled_heads(oracle):
    """The 1.5B-class layer shape (B=8, T=4096, H=32) through the C2 entry point; the oracle
    replays sampled (b, h) heads."""
    cfg = W.CONFIGS[1]
    inp = W.make_prefill_inputs(cfg, DEV)
    g = torch.Generator(device=DEV).manual_seed(8700)
    inp["uprime"] = (torch.randn(inp["r"].shape, generator=g, device=DEV) * 0.125).to(torch.bfloat16)
    y, s = _run(inp)
    for (b, h) in [(0, 0), (3, 17), (7, 31)]:
        sl = lambda t: f64(t[b:b + 1, :, h:h + 1])
        yo, so = oracle.prefill_c2(sl(inp["r"]), sl(inp["k"]), sl(inp["v"]), sl(inp["omega"]),
                                   sl(inp["uprime"]), f64(inp["state0"][b:b + 1, h:h + 1]))
        assert rel_err(y[b, :, h], yo[0, :, 0]) <= TOL[torch.bfloat16]
        assert rel_err(s[b, h], so[0, 0]) <= TOL[torch.bfloat16]


def test_c2_validation():
    inp = _problem(8800, B=1, T=40, H=2)
    L = bd.load()
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    y = torch.full_like(inp["r"], 3.0)
    ws = bd.new_workspace(bd.prefill_workspace_bytes(1, 40, 2, 64, torch.bfloat16, False), DEV)
    args = lambda up, yy: (vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), up,
                           vp(inp["state0"]), None, vp(yy), 1, 40, 2, 64, bd.WKV_BF16, None,
                           vp(ws), ws.numel(), None)
    assert L.wkv6c2_prefill(*args(None, y)) == bd.WKV_ERR_INVALID_ARG          # u' missing
    assert L.wkv6c2_prefill(*args(vp(y), y)) == bd.WKV_ERR_INVALID_ARG         # u' is y
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
    assert L.wkv6c2_prefill(*args(vp(inp["uprime"]), y)) == bd.WKV_OK


@pytest.mark.parametrize("omega_value", [-60.0, -12.0, 30.0])
def test_c2_saturated_and_slow_decay(oracle, omega_value):
    """1 - w at its ends: w = 1 to fp32 (1 - w ~ exp(omega), kept exact through the series
    for small exp(omega)) and w = 0 (1 - w = 1)."""
    inp = _problem(8900, B=1, T=150, H=2)
    inp["omega"] = torch.full_like(inp["v"], omega_value)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]
