"""C-ABI argument validation on a GPU: each bad call returns its status, launches nothing
and leaves every output untouched.  Calls go straight through ctypes with raw pointers."""
import ctypes
import os

import pytest
import torch

from linear_attention_rnn_finch_b200 import binding as bd

pytestmark = pytest.mark.gpu

B, T, H, D = 2, 40, 3, 64


def vp(t, offset=0):
    return None if t is None else ctypes.c_void_p(t.data_ptr() + offset)


@pytest.fixture()
def bufs():
    g = torch.Generator(device="cuda").manual_seed(9000)
    mk = lambda: (torch.randn(B, T, H, D, generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    d = dict(r=mk(), k=mk(), v=mk(), omega=mk(),
             u=torch.randn(H, D, generator=g, device="cuda"),
             s_in=torch.randn(B, H, D, D, generator=g, device="cuda") * 0.1,
             s_out=torch.full((B, H, D, D), 7.0, device="cuda"),
             y=torch.full((B, T, H, D), 3.0, device="cuda", dtype=torch.bfloat16),
             gamma=torch.ones(H * D, device="cuda"), beta=torch.zeros(H * D, device="cuda"))
    return d


def call(d, *, r=None, k=None, y=None, s_in=None, s_out=None, dims=(B, T, H, D), io=bd.WKV_BF16,
         ln=None, algo=0, ws=None, ws_bytes=0):
    L = bd.load()
    st = L.wkv6_prefill_algo(r or vp(d["r"]), k or vp(d["k"]), vp(d["v"]), vp(d["omega"]),
                             vp(d["u"]), s_in if s_in is not None else vp(d["s_in"]),
                             s_out if s_out is not None else vp(d["s_out"]),
                             y or vp(d["y"]), *dims, io, ln, algo, ws, ws_bytes, None)
    torch.cuda.synchronize()
    return st


def untouched(d):
    return bool((d["y"] == 3.0).all()) and bool((d["s_out"] == 7.0).all())


def test_valid_call_ok(bufs):
    ws = bd.new_workspace(bd.prefill_workspace_bytes(B, T, H, D, torch.bfloat16, False), "cuda")
    assert call(bufs, ws=vp(ws), ws_bytes=ws.numel()) == bd.WKV_OK
    assert not untouched(bufs)


def test_chunked_needs_workspace(bufs):
    assert call(bufs) == bd.WKV_ERR_WORKSPACE and untouched(bufs)
    assert call(bufs, algo=1) == bd.WKV_OK   # the recurrence needs none


def test_head_size_unsupported(bufs):
    assert call(bufs, dims=(B, T, H, 32)) == bd.WKV_ERR_UNSUPPORTED and untouched(bufs)


@pytest.mark.parametrize("dims", [(-1, T, H, D), (B, -5, H, D), (B, T, -2, D)])
def test_negative_sizes(bufs, dims):
    assert call(bufs, dims=dims) == bd.WKV_ERR_INVALID_ARG and untouched(bufs)


def test_null_input(bufs):
    L = bd.load()
    st = L.wkv6_prefill_algo(None, vp(bufs["k"]), vp(bufs["v"]), vp(bufs["omega"]), vp(bufs["u"]),
                             vp(bufs["s_in"]), vp(bufs["s_out"]), vp(bufs["y"]), B, T, H, D,
                             bd.WKV_BF16, None, 0, None, 0, None)
    assert st == bd.WKV_ERR_INVALID_ARG and untouched(bufs)


def test_misaligned_pointer(bufs):
    assert call(bufs, r=vp(bufs["r"], 2)) == bd.WKV_ERR_INVALID_ARG and untouched(bufs)


def test_host_pointer_rejected(bufs):
    host = bufs["r"].cpu().pin_memory()
    assert call(bufs, r=vp(host)) == bd.WKV_ERR_INVALID_ARG and untouched(bufs)


def test_output_overlapping_input(bufs):
    assert call(bufs, y=vp(bufs["r"])) == bd.WKV_ERR_INVALID_ARG
    assert bool((bufs["s_out"] == 7.0).all())


def test_state_partial_overlap(bufs):
    st = call(bufs, s_in=vp(bufs["s_out"]), s_out=vp(bufs["s_out"], 256))
    assert st == bd.WKV_ERR_INVALID_ARG and untouched(bufs)


def test_layernorm_needs_workspace(bufs):
    ln = bd._LN(bufs["gamma"].data_ptr(), bufs["beta"].data_ptr(), 1e-5)
    assert call(bufs, ln=ctypes.byref(ln)) == bd.WKV_ERR_WORKSPACE and untouched(bufs)
    need = bd.prefill_workspace_bytes(B, T, H, D, torch.bfloat16, True)
    ws = bd.new_workspace(need - 16, "cuda")
    assert call(bufs, ln=ctypes.byref(ln), ws=vp(ws), ws_bytes=need - 16) == bd.WKV_ERR_WORKSPACE
    ws = bd.new_workspace(need, "cuda")
    assert call(bufs, ln=ctypes.byref(ln), ws=vp(ws), ws_bytes=need) == bd.WKV_OK


def test_layernorm_bad_eps(bufs):
    ln = bd._LN(bufs["gamma"].data_ptr(), bufs["beta"].data_ptr(), 0.0)
    need = bd.prefill_workspace_bytes(B, T, H, D, torch.bfloat16, True)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert call(bufs, ln=ctypes.byref(ln), ws=vp(ws), ws_bytes=need) == bd.WKV_ERR_INVALID_ARG


def test_chunked_needs_bf16(bufs):
    assert call(bufs, io=bd.WKV_F32, algo=2) == bd.WKV_ERR_UNSUPPORTED and untouched(bufs)


def test_injected_launch_failure_raises(bufs, monkeypatch):
    monkeypatch.setenv("GOLDWKV_FAULT", "launch")
    with pytest.raises(bd.WkvError) as ei:
        bd.wkv6_prefill(bufs["r"], bufs["k"], bufs["v"], bufs["omega"], bufs["u"], bufs["s_in"])
    assert ei.value.status == bd.WKV_ERR_CUDA
    monkeypatch.delenv("GOLDWKV_FAULT")
    bd.wkv6_prefill(bufs["r"], bufs["k"], bufs["v"], bufs["omega"], bufs["u"], bufs["s_in"])


def test_decode_validation(bufs):
    L = bd.load()
    r = bufs["r"][:, 0].contiguous()
    state = bufs["s_in"].clone()
    y = torch.full((B, H, D), 5.0, device="cuda", dtype=torch.bfloat16)
    st = L.wkv6_decode_step(vp(r), vp(r), vp(r), vp(r), vp(bufs["u"]), vp(state), vp(y), B, H, 48,
                            bd.WKV_BF16, None, None, 0, None)
    assert st == bd.WKV_ERR_UNSUPPORTED
    st = L.wkv6_decode_step(vp(r), vp(r), vp(r), vp(r), vp(bufs["u"]), vp(state), vp(r), B, H, D,
                            bd.WKV_BF16, None, None, 0, None)
    assert st == bd.WKV_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(state, bufs["s_in"]) and bool((y == 5.0).all())


def test_chunked_wait_timeout_is_reported_and_context_survives(oracle, monkeypatch):
    """A zero spin budget makes the chunked kernel's first bounded wait expire: every CTA
    drains its in-flight copies, frees its tensor memory and returns; the workspace status
    word reports the timeout and the next call on the same context is correct."""
    from linear_attention_rnn_finch_b200 import workloads as W
    from tests.parity import TOL, f64, rel_err
    cfg = W.CONFIGS[1].with_(seed=9100)
    inp = W.make_prefill_inputs(cfg, "cuda", B=2, T=200)
    args = [inp[n] for n in ("r", "k", "v", "omega")]
    ws = bd.new_workspace(bd.prefill_workspace_bytes(2, 200, cfg.H, 64, torch.bfloat16, False), "cuda")
    monkeypatch.setenv("GOLDWKV_FAULT", "timeout0")
    bd.wkv6_prefill(*args, inp["u"], inp["state0"], algo="chunked", workspace=ws)
    assert bd.workspace_status(ws) == bd.WKV_ERR_TIMEOUT
    monkeypatch.delenv("GOLDWKV_FAULT")
    y, s = bd.wkv6_prefill(*args, inp["u"], inp["state0"], algo="chunked", workspace=ws)
    assert bd.workspace_status(ws) == bd.WKV_OK
    yo, so = oracle.prefill(*[f64(a) for a in args], f64(inp["u"]), f64(inp["state0"]))
    assert rel_err(y, yo) <= TOL[torch.bfloat16] and rel_err(s, so) <= TOL[torch.bfloat16]
