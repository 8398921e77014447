"""libgoldwkv_debug.so (built with -DGW_DEBUG): the chunked kernels check, on the device, the
coordinates of every copy and store and their threads' index ranges; a failed check sets
bit 1 of the call's status word and skips the access.  Small prefills through the debug
library's C ABI (the fast path alone, a sequence handed over to the level kernel, a forced
3-way sequence split) must leave the status word at zero and match the oracle."""
import ctypes

import pytest
import torch

from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import build as build_mod
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def dbg():
    if not build_mod.LIB_DEBUG.exists():
        pytest.fail(f"{build_mod.LIB_DEBUG} not built (python -m linear_attention_rnn_finch_b200.build --debug)")
    return bd.load(build_mod.LIB_DEBUG)


def vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def problem(seed, B, T, H, extreme=None):
    inp = W.make_prefill_inputs(W.CONFIGS[1].with_(seed=seed, H=H), DEV, B=B, T=T)
    if extreme is not None:   # tokens whose decay range the fast kernel hands over
        a, b_ = extreme
        om = inp["omega"].float()
        om[:, a:b_, H - 1, ::3] = 3.5
        inp["omega"] = om.to(torch.bfloat16)
    return inp


def run(L, inp):
    B, T, H, D = inp["r"].shape
    y = torch.full_like(inp["r"], 3.0)
    s = torch.full((B, H, D, D), 7.0, device=DEV)
    need = L.wkv6_prefill_workspace_bytes(B, T, H, D, bd.WKV_BF16, 0, 0)
    ws = bd.new_workspace(need, DEV)
    st = L.wkv6_prefill(vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), vp(inp["u"]),
                        vp(inp["state0"]), vp(s), vp(y), B, T, H, D, bd.WKV_BF16, None, vp(ws),
                        ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bd.WKV_OK
    torch.cuda.synchronize()
    return y, s, int(ws[:4].view(torch.int32).item())


@pytest.mark.parametrize("case", ["fast", "handover", "split3"])
def test_debug_build_checks_pass_and_results_match(dbg, oracle, monkeypatch, case):
    if case == "fast":
        inp = problem(9400, B=2, T=300, H=8)
    elif case == "handover":
        inp = problem(9401, B=2, T=700, H=2, extreme=(200, 330))
    else:
        monkeypatch.setenv("GOLDWKV_SEGMENTS", "3")
        inp = problem(9402, B=1, T=1100, H=2)
    y, s, word = run(dbg, inp)
    assert word == 0, f"status word {word}: bit 1 = a device-side check failed, bit 0 = timeout"
    yo, so = oracle.prefill(*[f64(inp[n]) for n in ("r", "k", "v", "omega", "u", "state0")])
    assert rel_err(y, yo) <= TOL[torch.bfloat16]
    assert rel_err(s, so) <= TOL[torch.bfloat16]
