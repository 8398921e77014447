"""wkv6_prefill_static: the prefill entry point that takes no workspace and allocates nothing.

Called straight through the C ABI with raw device pointers and compared with wkv6_prefill
(given a workspace of its own) on the same inputs, for two calls in a row that reuse the
built-in scratch: the second call hands one sequence over to the level-factorised kernel
through that scratch.  Also: sequences long enough to be split into segments, one whose
automatic split would not fit the scratch (served with a smaller split), and an expired
bounded wait reported by wkv6_prefill_static_status.  This file is named to be collected
last, and passes on its own too.
"""
import ctypes

import pytest
import torch

from linear_attention_rnn_finch_b200 import binding as bd
from linear_attention_rnn_finch_b200 import workloads as W
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def problem(seed, B, T, H, extreme=False):
    inp = W.make_prefill_inputs(W.CONFIGS[1].with_(seed=seed, H=H), DEV, B=B, T=T)
    if extreme:   # one chunk whose decay range the fast kernel cannot take
        om = inp["omega"].float()
        om[:, 128:192, 1, 5] = 6.0
        inp["omega"] = om.to(torch.bfloat16)
    return inp


def call_static(inp, y, s_out):
    B, T, H, D = inp["r"].shape
    return bd.load().wkv6_prefill_static(
        vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), vp(inp["u"]),
        vp(inp["state0"]), vp(s_out), vp(y), B, T, H, D, bd.WKV_BF16, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def call_with_workspace(inp):
    B, T, H, D = inp["r"].shape
    y = torch.empty_like(inp["r"])
    s = torch.empty(B, H, D, D, device=DEV)
    ws = bd.new_workspace(bd.prefill_workspace_bytes(B, T, H, D, torch.bfloat16, False), DEV)
    st = bd.load().wkv6_prefill(
        vp(inp["r"]), vp(inp["k"]), vp(inp["v"]), vp(inp["omega"]), vp(inp["u"]),
        vp(inp["state0"]), vp(s), vp(y), B, T, H, D, bd.WKV_BF16, None, vp(ws), ws.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bd.WKV_OK
    return y, s


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    first = problem(9300, B=2, T=1000, H=32)
    second = problem(9301, B=3, T=450, H=4, extreme=True)
    outs = []
    for inp in (first, second):   # enqueued back to back, no synchronisation between
        B, T, H, D = inp["r"].shape
        y = torch.full_like(inp["r"], 3.0)
        s = torch.full((B, H, D, D), 7.0, device=DEV)
        assert call_static(inp, y, s) == bd.WKV_OK
        outs.append((y, s))
    torch.cuda.synchronize()
    for inp, (y, s) in zip((first, second), outs):
        y_ref, s_ref = call_with_workspace(inp)
        torch.cuda.synchronize()
        assert rel_err(y, f64(y_ref)) <= TOL[torch.bfloat16]
        assert rel_err(s, f64(s_ref)) <= TOL[torch.bfloat16]


def test_no_device_memory_taken():
    inp = problem(9302, B=2, T=300, H=8)
    y = torch.empty_like(inp["r"])
    s = torch.empty(2, 8, 64, 64, device=DEV)
    assert call_static(inp, y, s) == bd.WKV_OK   # first call on this device: set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert call_static(inp, y, s) == bd.WKV_OK
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_sizes_beyond_the_scratch_are_rejected_untouched():
    # 8 x 64 = 512 (b,h) pairs need 512 hand-off states of 16 KB: more than 8 MiB
    B, T, H = 8, 3, 64
    need = bd.prefill_workspace_bytes(B, T, H, 64, torch.bfloat16, False)
    assert need > bd.STATIC_SCRATCH_BYTES
    inp = problem(9303, B=B, T=T, H=H)
    y = torch.full_like(inp["r"], 3.0)
    s = torch.full((B, H, 64, 64), 7.0, device=DEV)
    assert call_static(inp, y, s) == bd.WKV_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 3.0).all()) and bool((s == 7.0).all())
    # a problem that fits is served
    inp = problem(9304, B=1, T=T, H=H)
    y = torch.empty_like(inp["r"])
    s = torch.empty(1, H, 64, 64, device=DEV)
    assert call_static(inp, y, s) == bd.WKV_OK
    y_ref, s_ref = call_with_workspace(inp)
    torch.cuda.synchronize()
    assert rel_err(y, f64(y_ref)) <= TOL[torch.bfloat16]
    assert rel_err(s, f64(s_ref)) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("B,T,H", [(1, 16384, 4), (1, 65536, 8)])
def test_split_sequences_match_the_workspace_entry_point(B, T, H):
    """Few (b,h) pairs and long sequences: the chunked path cuts each sequence into
    segments.  At B=1, T=16384, H=4 the automatic split fits the scratch; at B=1, T=65536,
    H=8 its workspace (about 9.2 MiB) does not, and the call takes a smaller split."""
    auto = bd.prefill_workspace_bytes(B, T, H, 64, torch.bfloat16, False)
    unsplit = bd.prefill_workspace_bytes(B, T, H, 64, torch.bfloat16, False,
                                         algo="chunked_levels")
    assert auto > unsplit   # wkv6_prefill splits this problem
    if T == 65536:
        assert auto > bd.STATIC_SCRATCH_BYTES
    inp = problem(9305 + H, B=B, T=T, H=H)
    y = torch.full_like(inp["r"], 3.0)
    s = torch.full((B, H, 64, 64), 7.0, device=DEV)
    assert call_static(inp, y, s) == bd.WKV_OK
    assert bd.prefill_static_status() == bd.WKV_OK
    y_ref, s_ref = call_with_workspace(inp)
    torch.cuda.synchronize()
    assert rel_err(y, f64(y_ref)) <= TOL[torch.bfloat16]
    assert rel_err(s, f64(s_ref)) <= TOL[torch.bfloat16]


def test_expired_wait_is_reported_once_and_the_next_call_is_correct(monkeypatch):
    """A zero spin budget makes the first bounded wait of every CTA expire: the call still
    returns WKV_OK, the status query reports the timeout once and clears it, and the next
    call (normal budget) through the same scratch is correct."""
    inp = problem(9310, B=2, T=200, H=8)
    y = torch.empty_like(inp["r"])
    s = torch.empty(2, 8, 64, 64, device=DEV)
    assert bd.prefill_static_status() == bd.WKV_OK
    monkeypatch.setenv("GOLDWKV_FAULT", "timeout0")
    assert call_static(inp, y, s) == bd.WKV_OK
    assert bd.prefill_static_status() == bd.WKV_ERR_TIMEOUT
    assert bd.prefill_static_status() == bd.WKV_OK
    monkeypatch.delenv("GOLDWKV_FAULT")
    assert call_static(inp, y, s) == bd.WKV_OK
    assert bd.prefill_static_status() == bd.WKV_OK
    y_ref, s_ref = call_with_workspace(inp)
    torch.cuda.synchronize()
    assert rel_err(y, f64(y_ref)) <= TOL[torch.bfloat16]
    assert rel_err(s, f64(s_ref)) <= TOL[torch.bfloat16]
