"""The bf16 backward's stream ordering: its passes run on library side streams forked from
and joined back to the caller's stream by events, so to the caller a call is ordered on its
own stream like any other.

- on a stream of the caller's, with dy produced on that stream just before the call and the
  outputs reduced on it just after, the results equal a default-stream call bit for bit;
- captured into a CUDA graph (after a first call has made the side streams), a replay gives
  the same results as an eager call, bit for bit;
- two host threads calling at once, each on a stream of its own (the side streams and
  their events are shared per device), get the results of calls made one after another.
"""
import threading

import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, B=2, T=300, H=4):
    inp = W.make_prefill_inputs(W.CONFIGS[1].with_(seed=seed, H=H), DEV, B=B, T=T)
    g = torch.Generator(device=DEV).manual_seed(seed + 5)
    dy = torch.randn((B, T, H, 64), generator=g, device=DEV).to(torch.bfloat16)
    ds = torch.randn((B, H, 64, 64), generator=g, device=DEV) * 0.1
    return inp, dy, ds


def _call(inp, dy, ds, c2=False, stream=None):
    if c2:
        return gw.wkv6c2_backward(inp["r"], inp["k"], inp["v"], inp["omega"], inp["state0"], dy,
                                  ds, stream=stream)
    return gw.wkv6_backward(inp["r"], inp["k"], inp["v"], inp["omega"], inp["u"], inp["state0"],
                            dy, ds, stream=stream)


@pytest.mark.parametrize("c2", [False, True])
def test_backward_on_a_caller_stream(c2):
    inp, dy, ds = _inputs(7100)
    want = _call(inp, dy, ds, c2)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    dy_src = dy.float()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        dy_s = dy_src.to(torch.bfloat16)      # produced on s right before the call
        got = _call(inp, dy_s, ds, c2, stream=s)
        sums = [t.float().sum() for t in got if t is not None]   # consumed on s right after
    s.synchronize()
    for g, w in zip(got, want):
        if w is None:
            assert g is None
            continue
        assert torch.equal(g, w)
    for x, t in zip(sums, [t for t in want if t is not None]):
        assert torch.equal(x, t.float().sum())


@pytest.mark.parametrize("c2", [False, True])
def test_backward_graph_capture_replay(c2):
    inp, dy, ds = _inputs(7200)
    want = _call(inp, dy, ds, c2)   # also makes the side streams before the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    warm = torch.cuda.Stream()
    warm.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(warm):
        _call(inp, dy, ds, c2)
    torch.cuda.current_stream().wait_stream(warm)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        got = _call(inp, dy, ds, c2)
    graph.replay()
    torch.cuda.synchronize()
    for g, w in zip(got, want):
        if w is None:
            assert g is None
            continue
        assert torch.equal(g, w)
    del graph


@pytest.mark.parametrize("c2", [False, True])
def test_backward_two_host_threads(c2):
    problems = [_inputs(7300 + i) for i in range(2)]
    want = [_call(*p, c2) for p in problems]
    torch.cuda.synchronize()
    got, errors = [None, None], []

    def run(i):
        try:
            s = torch.cuda.Stream()
            outs = []
            with torch.cuda.stream(s):
                for _ in range(3):
                    outs.append(_call(*problems[i], c2, stream=s))
            s.synchronize()
            got[i] = outs
        except Exception as e:   # reported below, on the test's thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i in range(2):
        for outs in got[i]:
            for g, w in zip(outs, want[i]):
                if w is None:
                    assert g is None
                    continue
                assert torch.equal(g, w)
