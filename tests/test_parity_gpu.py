"""GPU parity: libgoldwkv (through its C ABI) against the fp64 oracle on seeded inputs.

Metric: max|gpu - oracle| / max|oracle| per tensor (y, final state); tolerance 1e-4 for
fp32 I/O and 5e-3 for bf16 I/O.  Small cases are compared element by element in full;
the full-size workloads are run whole on the GPU and compared on sampled heads / batch
rows, for which the oracle replays the whole sequence.
"""
import numpy as np
import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, oracle_heads, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16_ALGOS = ["chunked", "chunked_levels", "recurrent"]


def _run(inp, algo="auto", T=None, ln=False, state=True):
    T = inp["r"].shape[1] if T is None else T
    args = [inp[n][:, :T].contiguous() for n in ("r", "k", "v", "omega")]
    lnp = (inp["gamma"], inp["beta"], inp["eps"]) if ln else None
    y, s = gw.wkv6_prefill(*args, inp["u"], inp["state0"] if state else None, ln=lnp, algo=algo)
    torch.cuda.synchronize()
    return y, s


def _oracle_full(oracle, inp, T=None, ln=False, state=True):
    T = inp["r"].shape[1] if T is None else T
    a = [f64(inp[n][:, :T]) for n in ("r", "k", "v", "omega")]
    s0 = f64(inp["state0"]) if state else None
    if ln:
        y, s, _ = oracle.prefill_ln(*a, f64(inp["u"]), s0, f64(inp["gamma"]), f64(inp["beta"]),
                                    inp["eps"])
        return y, s
    return oracle.prefill(*a, f64(inp["u"]), s0)


# ----------------------------------------------------------------------------- small, full compare
@pytest.mark.parametrize("algo", ["auto", "recurrent"])
def test_tiny_f32(oracle, algo):
    cfg = W.CONFIGS[0]
    inp = W.make_prefill_inputs(cfg, DEV)
    y, s = _run(inp, algo)
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.float32]
    assert rel_err(s, so) <= TOL[torch.float32]


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 63, 64, 65, 100, 257])
def test_ragged_f32(oracle, T):
    cfg = W.CONFIGS[0].with_(B=2, H=3, state0="normal0.1", seed=7000 + T)
    inp = W.make_prefill_inputs(cfg, DEV, T=T)
    y, s = _run(inp)
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.float32]
    assert rel_err(s, so) <= TOL[torch.float32]


@pytest.mark.parametrize("algo", BF16_ALGOS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 513])
def test_bf16_small(oracle, algo, T):
    cfg = W.CONFIGS[1].with_(seed=7100 + T)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=T)
    inp["r"], inp["k"] = inp["r"][:, :, :4].contiguous(), inp["k"][:, :, :4].contiguous()
    inp["v"], inp["omega"] = inp["v"][:, :, :4].contiguous(), inp["omega"][:, :, :4].contiguous()
    inp["u"], inp["state0"] = inp["u"][:4].contiguous(), inp["state0"][:, :4].contiguous()
    y, s = _run(inp, algo)
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_zero_initial_state_is_none(oracle):
    cfg = W.CONFIGS[1].with_(seed=7200, state0="zero")
    inp = W.make_prefill_inputs(cfg, DEV, B=1, T=130)
    y1, s1 = _run(inp, state=False)
    y2, s2 = _run(inp, state=True)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_empty_sequence_passes_state_through():
    cfg = W.CONFIGS[1].with_(seed=7300)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=1)
    e = inp["r"][:, :0]
    _, s = gw.wkv6_prefill(e, e, e, e, inp["u"], inp["state0"])
    torch.cuda.synchronize()
    assert torch.equal(s, inp["state0"])
    _, s = gw.wkv6_prefill(e, e, e, e, inp["u"], None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(s) == 0


def test_state_in_place(oracle):
    cfg = W.CONFIGS[1].with_(seed=7400)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=77)
    yo, so = _oracle_full(oracle, inp)
    st = inp["state0"].clone()
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    y, s = gw.wkv6_prefill(*args, inp["u"], st, state_out=st)
    torch.cuda.synchronize()
    assert s is st
    assert rel_err(st, so) <= TOL[torch.bfloat16] and rel_err(y, yo) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("algo", BF16_ALGOS)
@pytest.mark.parametrize("omega_value", [-60.0, 30.0])
def test_decay_saturated(oracle, algo, omega_value):
    """w rounds to exactly 1 (omega=-60) or 0 (omega=+30) in fp32 and fp64 alike."""
    cfg = W.CONFIGS[1].with_(seed=7500)
    inp = W.make_prefill_inputs(cfg, DEV, B=1, T=150)
    inp["r"], inp["k"] = inp["r"][:, :, :3].contiguous(), inp["k"][:, :, :3].contiguous()
    inp["v"] = inp["v"][:, :, :3].contiguous()
    inp["omega"] = torch.full_like(inp["v"], omega_value)
    inp["u"], inp["state0"] = inp["u"][:3].contiguous(), inp["state0"][:, :3].contiguous()
    y, s = _run(inp, algo)
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("extreme_from", [0, 64, 130, 300])
def test_handoff_mid_sequence(oracle, extreme_from):
    """Mild decays up to token `extreme_from`, then some channels with w ~ 0: the fast
    kernel takes the first chunks and hands the rest (and its state) to the level kernel."""
    cfg = W.CONFIGS[1].with_(seed=7550 + extreme_from)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=400)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n][:, :, :4].contiguous()
    inp["u"], inp["state0"] = inp["u"][:4].contiguous(), inp["state0"][:, :4].contiguous()
    om = inp["omega"].float()
    om[:, extreme_from:, :, ::3] = 3.5          # exp(-exp(3.5)) ~ 4e-15 per token
    inp["omega"] = om.to(torch.bfloat16)
    y, s = _run(inp, "chunked")
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_isolated_extreme_chunk(oracle):
    """A single chunk with an extreme decay in the middle of a mild sequence."""
    cfg = W.CONFIGS[1].with_(seed=7560)
    inp = W.make_prefill_inputs(cfg, DEV, B=1, T=320)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n][:, :, :2].contiguous()
    inp["u"], inp["state0"] = inp["u"][:2].contiguous(), inp["state0"][:, :2].contiguous()
    om = inp["omega"].float()
    om[:, 128:192, 1, 5] = 6.0
    inp["omega"] = om.to(torch.bfloat16)
    for algo in ("chunked", "chunked_levels"):
        y, s = _run(inp, algo)
        yo, so = _oracle_full(oracle, inp)
        assert rel_err(y, yo) <= TOL[torch.bfloat16], algo
        assert rel_err(s, so) <= TOL[torch.bfloat16], algo


# ----------------------------------------------------------------------------- sequence split
def _small(seed, B, T, H):
    inp = W.make_prefill_inputs(W.CONFIGS[1].with_(seed=seed), DEV, B=B, T=T)
    for n in ("r", "k", "v", "omega"):
        inp[n] = inp[n][:, :, :H].contiguous()
    inp["u"], inp["state0"] = inp["u"][:H].contiguous(), inp["state0"][:, :H].contiguous()
    return inp


@pytest.mark.parametrize("P", [2, 3, 6])
@pytest.mark.parametrize("case", ["mild", "zero_state", "handoff_late", "ragged"])
def test_sequence_split(oracle, monkeypatch, P, case):
    """Segments of one sequence on different CTAs: the state pre-pass and carry give each
    segment its incoming state; the result must match the unsplit oracle run."""
    monkeypatch.setenv("GOLDWKV_SEGMENTS", str(P))
    T = {"ragged": 1001}.get(case, 1024)
    inp = _small(7700 + P, B=2, T=T, H=3)
    if case == "handoff_late":   # an extreme chunk inside a later segment
        om = inp["omega"].float()
        om[:, 830:900, 1, 5] = 6.0
        inp["omega"] = om.to(torch.bfloat16)
    state = case != "zero_state"
    nc = (T + 63) // 64
    seg = (nc + P - 1) // P
    hand = lambda units: 256 + ((units * 4 + 255) // 256) * 256 + units * 16384
    assert gw.prefill_workspace_bytes(2, T, 3, 64, torch.bfloat16, False) == \
        hand(6 * P) + 6 * (P - 1) * (4096 + 64) * 4, "the split was not taken"
    assert (P - 1) * seg < nc
    y, s = _run(inp, "chunked", state=state)
    yo, so = _oracle_full(oracle, inp, state=state)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("omega_value", [-60.0, 30.0])
def test_sequence_split_saturated_decay(oracle, monkeypatch, omega_value):
    """w = 1 everywhere (segment decay product 1: the whole state carries) and w = 0 (the
    product underflows to 0: nothing carries)."""
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "4")
    inp = _small(7800, B=1, T=1280, H=2)
    inp["omega"] = torch.full_like(inp["v"], omega_value)
    y, s = _run(inp, "chunked")
    yo, so = _oracle_full(oracle, inp)
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_sequence_split_matches_unsplit(monkeypatch):
    """Split and unsplit runs of the same problem agree to the tolerance (they differ only
    in rounding order)."""
    inp = _small(7810, B=2, T=2048, H=4)
    y1, s1 = _run(inp, "chunked")
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "4")
    y4, s4 = _run(inp, "chunked")
    dy = (y1.float() - y4.float()).abs().max().item() / y1.float().abs().max().item()
    ds = (s1 - s4).abs().max().item() / s1.abs().max().item()
    assert dy <= TOL[torch.bfloat16] and ds <= TOL[torch.bfloat16], (dy, ds)


def test_deterministic():
    cfg = W.CONFIGS[1].with_(seed=7600)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=300)
    y1, s1 = _run(inp)
    y2, s2 = _run(inp)
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


# ------------------------------------------------------------------------------- full workloads
SAMPLE_HEADS_1P5B = [(0, 0), (0, 31), (1, 7), (3, 16), (5, 25), (7, 0), (7, 31), (6, 12)]


@pytest.fixture(scope="module")
def cfg1_inputs():
    return W.make_prefill_inputs(W.CONFIGS[1], DEV)


@pytest.mark.parametrize("algo", BF16_ALGOS)
def test_prefill_1p5b_layer_full(oracle, cfg1_inputs, algo):
    inp = cfg1_inputs
    y, s = _run(inp, algo)
    ref = oracle_heads(oracle, inp, SAMPLE_HEADS_1P5B)
    ey = max(rel_err(y[b, :, h], ref[(b, h)][0]) for (b, h) in SAMPLE_HEADS_1P5B)
    es = max(rel_err(s[b, h], ref[(b, h)][1]) for (b, h) in SAMPLE_HEADS_1P5B)
    assert ey <= TOL[torch.bfloat16], ey
    assert es <= TOL[torch.bfloat16], es


@pytest.fixture(scope="module")
def cfg2_inputs():
    return W.make_prefill_inputs(W.CONFIGS[2], DEV)


def test_prefill_long_context_single_and_split(oracle, cfg2_inputs):
    inp = cfg2_inputs
    heads = [(0, 0), (0, 37)]
    ref = oracle_heads(oracle, inp, heads)
    y, s = _run(inp)
    # the same sequence as 4 consecutive 65536-token calls passing the state through
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    st = None
    ys = torch.empty_like(y)
    for c in range(4):
        sl = slice(c * 65536, (c + 1) * 65536)
        part = [a[:, sl].contiguous() for a in args]
        yc, st = gw.wkv6_prefill(*part, inp["u"], st)
        ys[:, sl] = yc
    torch.cuda.synchronize()
    for (b, h) in heads:
        for yy, ss in ((y, s), (ys, st)):
            assert rel_err(yy[b, :, h], ref[(b, h)][0]) <= TOL[torch.bfloat16]
            assert rel_err(ss[b, h], ref[(b, h)][1]) <= TOL[torch.bfloat16]
    # single vs split on every head: both are the same recurrence
    d = (y.float() - ys.float()).abs().max().item() / max(1e-30, y.float().abs().max().item())
    assert d <= TOL[torch.bfloat16], d


def test_decode_100_steps(oracle):
    cfg = W.CONFIGS[3]
    inp = W.make_decode_inputs(cfg, DEV)
    rows = [0, 77, 255]
    state = inp["state0"].clone()
    st_o = f64(inp["state0"][rows])
    u = f64(inp["u"])
    worst_y = 0.0
    for step in range(cfg.steps):
        a = [inp[n][step] for n in ("r", "k", "v", "omega")]
        y = gw.wkv6_decode_step(*a, inp["u"], state)
        yo, st_o = oracle.decode_step(*[f64(x[rows]) for x in a], u, st_o)
        worst_y = max(worst_y, rel_err(y[rows], yo))
    torch.cuda.synchronize()
    assert worst_y <= TOL[torch.bfloat16], worst_y
    assert rel_err(state[rows], st_o) <= TOL[torch.bfloat16]


def test_decode_with_layernorm(oracle):
    cfg = W.CONFIGS[3].with_(seed=7700)
    inp = W.make_decode_inputs(cfg, DEV, B=6, steps=3)
    H, D = cfg.H, cfg.D
    g = torch.Generator(device=DEV).manual_seed(7701)
    gamma = 1 + 0.1 * torch.randn(H * D, generator=g, device=DEV)
    beta = 0.1 * torch.randn(H * D, generator=g, device=DEV)
    state = inp["state0"].clone()
    st_o = f64(inp["state0"])
    for step in range(3):
        a = [inp[n][step] for n in ("r", "k", "v", "omega")]
        y = gw.wkv6_decode_step(*a, inp["u"], state, ln=(gamma, beta, 1e-5))
        yo, st_o = oracle.decode_step(*[f64(x) for x in a], f64(inp["u"]), st_o)
        ylo = oracle.layernorm(yo.reshape(6, H * D), f64(gamma), f64(beta), 1e-5).reshape(6, H, D)
        assert rel_err(y, ylo) <= TOL[torch.bfloat16]
    assert rel_err(state, st_o) <= TOL[torch.bfloat16]


@pytest.fixture(scope="module")
def cfg4_inputs():
    return W.make_prefill_inputs(W.CONFIGS[4], DEV)


@pytest.mark.parametrize("algo", BF16_ALGOS)
def test_decay_extreme_layernorm_full(oracle, cfg4_inputs, algo):
    inp = cfg4_inputs
    y, s = _run(inp, algo, ln=True)
    b = 1
    one = {n: inp[n][b:b + 1] for n in ("r", "k", "v", "omega", "state0")}
    one.update(u=inp["u"], gamma=inp["gamma"], beta=inp["beta"], eps=inp["eps"])
    yo, so = _oracle_full(oracle, one, ln=True)
    assert rel_err(y[b:b + 1], yo) <= TOL[torch.bfloat16]
    assert rel_err(s[b:b + 1], so) <= TOL[torch.bfloat16]


def test_layernorm_small_f32(oracle):
    cfg = W.CONFIGS[4].with_(io="f32", seed=7800)
    inp = W.make_prefill_inputs(cfg, DEV, B=2, T=70)
    y, s = _run(inp, ln=True)
    yo, so = _oracle_full(oracle, inp, ln=True)
    assert rel_err(y, yo) <= TOL[torch.float32]
    assert rel_err(s, so) <= TOL[torch.float32]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_layernorm_one_kernel_reused_workspace(oracle, dtype):
    """Decode with LayerNorm runs as one kernel: the last CTA of each batch row normalises
    it and resets the row's counter.  One zero-filled workspace serves 6 steps in a row
    (B=5 rows, H=12 heads, so rows do not fill a wave evenly), its counters are zero after
    each step, and y and the state match the oracle at every step."""
    cfg = W.CONFIGS[3].with_(seed=9500, B=5, H=12, io="f32" if dtype == torch.float32 else "bf16")
    inp = W.make_decode_inputs(cfg, "cuda", steps=6)
    B, H, D = 5, 12, 64
    g = torch.Generator(device="cuda").manual_seed(9501)
    gamma = 1.0 + 0.1 * torch.randn(H * D, generator=g, device="cuda")
    beta = 0.1 * torch.randn(H * D, generator=g, device="cuda")
    ws = gw.new_workspace(gw.decode_workspace_bytes(B, H, D, dtype, True), "cuda")
    state = inp["state0"].clone()
    st_o = f64(inp["state0"])
    for t in range(6):
        a = [inp[n][t] for n in ("r", "k", "v", "omega")]
        y = gw.wkv6_decode_step(*a, inp["u"], state, ln=(gamma, beta, 1e-5), workspace=ws)
        torch.cuda.synchronize()
        assert int(ws[:4 * B].view(torch.int32).abs().sum()) == 0
        yo, st_o = oracle.decode_step(*[f64(x) for x in a], f64(inp["u"]), st_o)
        yo = oracle.layernorm(yo.reshape(B, H * D), f64(gamma), f64(beta), 1e-5).reshape(B, H, D)
        assert rel_err(y, yo) <= TOL[dtype]
        assert rel_err(state, st_o) <= TOL[dtype]
