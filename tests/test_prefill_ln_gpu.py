"""Prefill with LayerNorm (bf16 chunked path), against the fp64 oracle.

The recurrence kernels stage each token's fp32 rows, normalised over all H*64 channels by
extra CTAs of the level kernel's launch when the recurrence's CTAs leave room on the device
and H <= 32, else by a second kernel (the last cases here force that: more (b,h) units than
the device holds at once, or H > 32).  These cases cover each way a token chunk's rows can
be produced:
the fast kernel alone, the level-factorised kernel alone, a hand-over from one to the other
in the middle of a sequence (so one chunk's heads come from both kernels), a forced sequence
split, ragged tails, one head, odd head counts, Finch-C2's form, and repeated calls on one
workspace, one of them cut short by an expired bounded wait.
"""
import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def problem(seed, B, T, H, cfg=1, extreme=None):
    inp = W.make_prefill_inputs(W.CONFIGS[cfg].with_(seed=seed, H=H, ln=True), DEV, B=B, T=T)
    if extreme is not None:   # tokens whose decay range the fast kernel hands over
        a, b_ = extreme
        om = inp["omega"].float()
        om[:, a:b_, H - 1, ::3] = 3.5
        inp["omega"] = om.to(torch.bfloat16)
    return inp


def run(inp, algo="auto", workspace=None):
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    y, s = gw.wkv6_prefill(*args, inp["u"], inp["state0"], ln=(inp["gamma"], inp["beta"], inp["eps"]),
                           algo=algo, workspace=workspace)
    torch.cuda.synchronize()
    return y, s


def oracle_ln(oracle, inp):
    a = [f64(inp[n]) for n in ("r", "k", "v", "omega", "u", "state0")]
    y, s, _ = oracle.prefill_ln(*a, f64(inp["gamma"]), f64(inp["beta"]), inp["eps"])
    return y, s


def check(oracle, inp, y, s):
    yo, so = oracle_ln(oracle, inp)
    assert torch.isfinite(y.float()).all()
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 640])
@pytest.mark.parametrize("algo", ["chunked", "chunked_levels"])
def test_prefill_ln_ragged(oracle, T, algo):
    inp = problem(9500 + T, B=2, T=T, H=3)
    check(oracle, inp, *run(inp, algo))


@pytest.mark.parametrize("H", [1, 2, 5, 32])
def test_prefill_ln_head_counts(oracle, H):
    inp = problem(9520 + H, B=1, T=150, H=H)
    check(oracle, inp, *run(inp))


def test_prefill_ln_handover_mid_sequence(oracle):
    # head H-1 hands over to the level kernel at token 200's chunk; the others stay fast
    inp = problem(9530, B=2, T=700, H=4, extreme=(200, 330))
    check(oracle, inp, *run(inp))


def test_prefill_ln_all_extreme(oracle):
    inp = problem(9531, B=2, T=300, H=4, cfg=4)
    check(oracle, inp, *run(inp))


def test_prefill_ln_sequence_split(oracle, monkeypatch):
    monkeypatch.setenv("GOLDWKV_SEGMENTS", "3")
    inp = problem(9532, B=1, T=1100, H=3, extreme=(500, 560))
    check(oracle, inp, *run(inp))


def test_prefill_ln_c2(oracle):
    inp = problem(9533, B=2, T=190, H=3)
    g = torch.Generator(device=DEV).manual_seed(9534)
    up = (0.125 * torch.randn(inp["r"].shape, generator=g, device=DEV)).to(torch.bfloat16)
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    y, s = gw.wkv6c2_prefill(*args, up, inp["state0"], ln=(inp["gamma"], inp["beta"], inp["eps"]))
    torch.cuda.synchronize()
    a = [f64(x) for x in (*args, up, inp["state0"])]
    yo, so, _ = oracle.prefill_c2_ln(*a, f64(inp["gamma"]), f64(inp["beta"]), inp["eps"])
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]


def test_prefill_ln_reused_workspace_after_expired_wait(oracle, monkeypatch):
    inp = problem(9535, B=2, T=330, H=4, extreme=(100, 140))
    B, T, H, D = inp["r"].shape
    ws = bd.new_workspace(bd.prefill_workspace_bytes(B, T, H, D, torch.bfloat16, True), DEV)
    y1, s1 = run(inp, workspace=ws)
    # every bounded wait expires at once: the call reports it and leaves counters counted
    monkeypatch.setenv("GOLDWKV_FAULT", "timeout0")
    run(inp, workspace=ws)
    monkeypatch.delenv("GOLDWKV_FAULT")
    assert bd.workspace_status(ws) == bd.WKV_ERR_TIMEOUT
    for _ in range(2):
        y, s = run(inp, workspace=ws)
        assert bd.workspace_status(ws) == bd.WKV_OK
        assert torch.equal(y, y1) and torch.equal(s, s1)
    check(oracle, inp, y1, s1)


@pytest.mark.parametrize("algo", ["chunked", "chunked_levels"])
@pytest.mark.parametrize("B,H,T", [(5, 32, 130), (1, 40, 70)])
def test_prefill_ln_second_pass(oracle, B, H, T, algo):
    """160 (b,h) units fill every SM (no room for the normalising CTAs), or 40 heads (rows
    wider than the in-launch LayerNorm takes): the staged rows go through the second kernel."""
    inp = problem(9700 + B * H + T, B=B, T=T, H=H)
    check(oracle, inp, *run(inp, algo))


def test_prefill_ln_graph_capture():
    """The in-launch LayerNorm is a cooperative launch: captured into a CUDA graph and replayed,
    the call gives what an eager call gives, bit for bit."""
    inp = problem(9800, B=2, T=200, H=4)
    want, _ = run(inp)
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    ln = (inp["gamma"], inp["beta"], inp["eps"])
    warm = torch.cuda.Stream()
    warm.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(warm):
        gw.wkv6_prefill(*args, inp["u"], inp["state0"], ln=ln)
    torch.cuda.current_stream().wait_stream(warm)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        got, _ = gw.wkv6_prefill(*args, inp["u"], inp["state0"], ln=ln)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    del graph
