"""GPU parity of the sequence-parallel steps (wkv6_segment_summary, wkv6_segment_carry) and
of their composition: a sequence cut into P spans, each summarised, the states carried, each
span prefilled from its incoming state -- what P ranks do, run here one span after another
on one GPU -- against the oracle's single run and against one wkv6_prefill call."""
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


def _inputs(seed, B, T, H, extreme=False):
    inp = W.make_prefill_inputs(W.CONFIGS[1].with_(seed=seed, H=H), DEV, B=B, T=T)
    if extreme:   # strong decays: the summary takes any decay (factors <= 1)
        om = inp["omega"].float()
        om[:, :, 0, ::2] = 3.0
        inp["omega"] = om.to(torch.bfloat16)
    return inp


@pytest.mark.parametrize("extreme", [False, True])
def test_summary_is_the_state_from_zero_and_the_decay_sum(oracle, extreme):
    B, T, H = 2, 320, 4
    inp = _inputs(9700 + extreme, B, T, H, extreme)
    s_loc, g = bd.segment_summary(inp["k"], inp["v"], inp["omega"])
    torch.cuda.synchronize()
    f = lambda n: f64(inp[n])
    _, s_ref = oracle.prefill(np.zeros((B, T, H, 64)), f("k"), f("v"), f("omega"),
                              np.zeros((H, 64)), None)
    g_ref = (-np.exp(f("omega"))).sum(axis=1) / np.log(2.0)
    assert rel_err(s_loc, s_ref) <= TOL[torch.bfloat16]
    assert np.abs(f64(g) - g_ref).max() <= 1e-5 * np.abs(g_ref).max()


@pytest.mark.parametrize("P", [2, 4])
def test_spans_carried_equal_the_single_run(oracle, P):
    B, T_span, H = 2, 256, 4
    inp = _inputs(9710 + P, B, P * T_span, H)
    names = ("r", "k", "v", "omega")
    spans = [{n: inp[n][:, p * T_span:(p + 1) * T_span].contiguous() for n in names}
             for p in range(P)]
    summ = [bd.segment_summary(sp["k"], sp["v"], sp["omega"]) for sp in spans]
    s_in = bd.segment_carry(torch.stack([x[0] for x in summ]), torch.stack([x[1] for x in summ]),
                            inp["state0"])
    ys = [gw.wkv6_prefill(*(sp[n] for n in names), inp["u"], s_in[p].contiguous())[0]
          for p, sp in enumerate(spans)]
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1)
    yo, so = oracle.prefill(*[f64(inp[n]) for n in names], f64(inp["u"]), f64(inp["state0"]))
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s_in[P], so) <= TOL[torch.bfloat16]
    y1, s1 = gw.wkv6_prefill(*(inp[n] for n in names), inp["u"], inp["state0"])
    torch.cuda.synchronize()
    assert rel_err(y, f64(y1)) <= TOL[torch.bfloat16]


def test_carry_matches_its_definition():
    P, B, H = 3, 2, 3
    g = torch.Generator(device=DEV).manual_seed(9720)
    s_loc = torch.randn((P, B, H, 64, 64), generator=g, device=DEV)
    dec = -3.0 * torch.rand((P, B, H, 64), generator=g, device=DEV)
    s0 = torch.randn((B, H, 64, 64), generator=g, device=DEV)
    out = bd.segment_carry(s_loc, dec, s0)
    torch.cuda.synchronize()
    s = f64(s0)
    assert np.array_equal(f64(out[0]), s)
    for p in range(P):
        s = np.exp2(f64(dec[p]))[..., None] * s + f64(s_loc[p])
        assert np.abs(f64(out[p + 1]) - s).max() <= 1e-5 * np.abs(s).max()


def test_summary_argument_checks():
    L = bd.load()
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = _inputs(9730, 1, 100, 2)   # T not a multiple of 64
    s = torch.full((1, 2, 64, 64), 7.0, device=DEV)
    g = torch.full((1, 2, 64), 7.0, device=DEV)
    ws = bd.new_workspace(256, DEV)
    st = L.wkv6_segment_summary(vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), 0, vp(s), vp(g),
                                1, 100, 2, 64, bd.WKV_BF16, vp(ws), 256, stream)
    assert st == bd.WKV_ERR_UNSUPPORTED
    st = L.wkv6_segment_summary(vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), 0, vp(inp["k"]),
                                vp(g), 1, 64, 2, 64, bd.WKV_BF16, vp(ws), 256, stream)
    assert st == bd.WKV_ERR_INVALID_ARG   # output on top of an input
    torch.cuda.synchronize()
    assert bool((s == 7.0).all()) and bool((g == 7.0).all())
    # no tokens: the zero state and no decay
    st = L.wkv6_segment_summary(None, None, None, 0, vp(s), vp(g), 1, 0, 2, 64, bd.WKV_BF16,
                                None, 0, stream)
    assert st == bd.WKV_OK
    torch.cuda.synchronize()
    assert bool((s == 0).all()) and bool((g == 0).all())
