"""GPU parity of base Finch's output stage (wkv6_prefill_gn / wkv6_decode_step_gn) against
the fp64 oracle: the base recurrence, then GroupNorm over each head's 64 channels of each
token with a per-channel affine, then the output gate -- the two pieces Finch-C2 removes.

Covered: the chunked bf16 path (fast kernel, level kernel after a hand-over, the sequence
split with and without a hand-over), the fp32 recurrence, the gate absent, the decode step
in both dtypes, and the argument checks.
"""
import ctypes

import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
GN_EPS = 64e-5   # a per-head eps as base Finch models use it; any eps > 0 is accepted


def _problem(seed, B, T, H, dtype=torch.bfloat16, cfg=1, gate=True):
    inp = W.make_prefill_inputs(W.CONFIGS[cfg].with_(seed=seed, H=H), DEV, B=B, T=T)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n].float().to(dtype).contiguous()
    g = torch.Generator(device=DEV).manual_seed(seed + 7)
    inp["gamma"] = 1.0 + 0.2 * torch.randn(H * 64, generator=g, device=DEV)
    inp["beta"] = 0.1 * torch.randn(H * 64, generator=g, device=DEV)
    # a gate in (0, 1) x 2, as a sigmoid- or SiLU-style activation would give
    inp["gate"] = (2.0 * torch.rand((B, T, H, 64), generator=g, device=DEV)).to(dtype) \
        if gate else None
    return inp


def _run(inp, eps=GN_EPS):
    a = [inp[n] for n in ("r", "k", "v", "omega", "u")]
    y, s = gw.wkv6_prefill_gn(*a, inp["state0"], gn=(inp["gamma"], inp["beta"], eps, inp["gate"]))
    torch.cuda.synchronize()
    return y, s


def _oracle(oracle, inp, eps=GN_EPS):
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega", "u")]
    gate = None if inp["gate"] is None else f64(inp["gate"])
    yo, so, _ = oracle.prefill_gn(*a, f64(inp["state0"]), f64(inp["gamma"]), f64(inp["beta"]),
                                  eps, gate)
    return yo, so


@pytest.mark.parametrize("T", [1, 64, 200, 513])
def test_gn_chunked(oracle, T):
    inp = _problem(9500 + T, B=2, T=T, H=4)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_gn_without_gate(oracle):
    inp = _problem(9520, B=2, T=130, H=3, gate=False)
    y, s = _run(inp, eps=1e-5)
    yo, so = _oracle(oracle, inp, eps=1e-5)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_gn_level_kernel_hand_over(oracle):
    inp = _problem(9530, B=2, T=300, H=3)
    om = inp["omega"].float()
    om[:, 140:, 1, ::3] = 3.5     # decay range the fast kernel hands to the level kernel
    inp["omega"] = om.to(torch.bfloat16)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("extreme_from", [0, 700])
def test_gn_split_with_hand_over(oracle, monkeypatch, extreme_from):
    """Sequence split into 3 segments with a hand-over to the level kernel in the first or
    the last segment: the GroupNorm pass sees rows from both kernels."""
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "3")
    inp = _problem(9545 + extreme_from, B=1, T=1100, H=2)
    om = inp["omega"].float()
    om[:, extreme_from:extreme_from + 90, 1, ::4] = 3.5
    inp["omega"] = om.to(torch.bfloat16)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_gn_sequence_split(oracle, monkeypatch):
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "3")
    inp = _problem(9540, B=1, T=1100, H=2)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_gn_full_layer_shape_sampled_heads(oracle):
    """B8 T4096 H32 bf16 with the gate, as bench.py times it; three heads through the oracle
    (the GroupNorm is local to a head, so a head's rows check on their own)."""
    cfg = W.CONFIGS[1]
    inp = _problem(cfg.seed, B=cfg.B, T=cfg.T, H=cfg.H)
    y, s = _run(inp)
    for b, h in ((0, 0), (3, 17), (7, 31)):
        one = {n: inp[n][b:b + 1, :, h:h + 1] for n in ("r", "k", "v", "omega", "gate")}
        a = [f64(one[n]) for n in ("r", "k", "v", "omega")]
        hs = slice(64 * h, 64 * h + 64)
        yo, so, _ = oracle.prefill_gn(*a, f64(inp["u"][h:h + 1]),
                                      f64(inp["state0"][b:b + 1, h:h + 1]),
                                      f64(inp["gamma"][hs]), f64(inp["beta"][hs]), GN_EPS,
                                      f64(one["gate"]))
        assert rel_err(y[b:b + 1, :, h:h + 1], yo) <= TOL[torch.bfloat16]
        assert rel_err(s[b:b + 1, h:h + 1], so) <= TOL[torch.bfloat16]


def test_gn_fp32_recurrence(oracle):
    inp = _problem(9550, B=2, T=150, H=2, dtype=torch.float32, cfg=0)
    y, s = _run(inp)
    yo, so = _oracle(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.float32]
    assert rel_err(s, so) <= TOL[torch.float32]


def test_gn_rows_are_normalised_before_the_gate(oracle):
    """With gamma = 1, beta = 0 and no gate each head's 64 outputs of each token have mean 0
    and (biased) variance var/(var + eps), which is 1 to fp32 precision when eps is far
    below every row's variance (here >= 1e-7 against eps = 1e-12): a property of any
    correct kernel, at any size."""
    inp = _problem(9560, B=2, T=257, H=4, dtype=torch.float32, cfg=0, gate=False)
    inp["gamma"] = torch.ones_like(inp["gamma"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    y, _ = _run(inp, eps=1e-12)
    yd = y.double()
    assert yd.mean(-1).abs().max().item() < 1e-5
    assert ((yd.var(-1, unbiased=False) - 1.0).abs() < 1e-4).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gn_decode_steps(oracle, dtype):
    g = torch.Generator(device=DEV).manual_seed(9600)
    B, H, D, steps = 16, 4, 64, 4
    mk = lambda s_: (torch.randn((B, H, D), generator=g, device=DEV) * s_).to(dtype)
    u = torch.randn((H, D), generator=g, device=DEV) * 0.5
    gamma = 1.0 + 0.2 * torch.randn(H * D, generator=g, device=DEV)
    beta = 0.1 * torch.randn(H * D, generator=g, device=DEV)
    state = torch.randn((B, H, D, D), generator=g, device=DEV) * 0.1
    s_ref = f64(state)
    for _ in range(steps):
        r, k, v = mk(0.125), mk(0.125), mk(0.125)
        om = (-6.0 + 7.0 * torch.rand((B, H, D), generator=g, device=DEV)).to(dtype)
        gate = (2.0 * torch.rand((B, H, D), generator=g, device=DEV)).to(dtype)
        y = gw.wkv6_decode_step_gn(r, k, v, om, u, state, gn=(gamma, beta, GN_EPS, gate))
        torch.cuda.synchronize()
        y_raw, s_ref = oracle.decode_step(f64(r), f64(k), f64(v), f64(om), f64(u), s_ref)
        yo = oracle.groupnorm_gate(y_raw, f64(gamma), f64(beta), GN_EPS, f64(gate))
        assert rel_err(y, yo) <= TOL[dtype]
    assert rel_err(state, s_ref) <= TOL[dtype]


def _raw_prefill_gn(inp, gn_struct, y, s):
    B, T, H, D = inp["r"].shape
    ws = bd.new_workspace(bd.prefill_workspace_bytes(B, T, H, D, inp["r"].dtype, True), DEV)
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return bd.load().wkv6_prefill_gn(
        vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), vp(inp["u"]),
        vp(inp["state0"]), vp(s), vp(y), B, T, H, D, bd._io(inp["r"].dtype),
        None if gn_struct is None else ctypes.byref(gn_struct), vp(ws), ws.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_gn_argument_checks():
    inp = _problem(9700, B=1, T=70, H=2)
    y = torch.full_like(inp["r"], 3.0)
    s = torch.full((1, 2, 64, 64), 7.0, device=DEV)
    gp = lambda t: t.data_ptr()
    ok = bd._GN(gp(inp["gamma"]), gp(inp["beta"]), 1e-5, gp(inp["gate"]))
    bad_eps = bd._GN(gp(inp["gamma"]), gp(inp["beta"]), 0.0, gp(inp["gate"]))
    no_beta = bd._GN(gp(inp["gamma"]), None, 1e-5, None)
    gate_on_y = bd._GN(gp(inp["gamma"]), gp(inp["beta"]), 1e-5, gp(y))
    for gn in (None, bad_eps, no_beta, gate_on_y):
        assert _raw_prefill_gn(inp, gn, y, s) == bd.WKV_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((y == 3.0).all()) and bool((s == 7.0).all())   # nothing launched
    assert _raw_prefill_gn(inp, ok, y, s) == bd.WKV_OK
