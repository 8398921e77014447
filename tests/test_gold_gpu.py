"""GPU parity of GOLD key compression and TokenCat decompression (gold_compress /
gold_decompress) against the fp64 oracle: c = x W_KD and RMSNorm(concat(x0, c) W_KU).

Ragged row counts, the chained call (decompressing the GPU's own compressed cache), the
1.5B-model shape (D = 2048, Dc = 128, B8 x T4096 tokens) on sampled rows, and the argument
checks.
"""
import ctypes

import pytest
import torch

import linear_attention_rnn_finch_b200 as gw
from linear_attention_rnn_finch_b200 import binding as bd
from tests.parity import TOL, f64, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = TOL[torch.bfloat16]


def _weights(seed, D, Dc):
    g = torch.Generator(device=DEV).manual_seed(seed)
    w_kd = (torch.randn((Dc, D), generator=g, device=DEV) / D ** 0.5).to(torch.bfloat16)
    w_ku = (torch.randn((D, D + Dc), generator=g, device=DEV) / (D + Dc) ** 0.5).to(torch.bfloat16)
    gamma = 1.0 + 0.2 * torch.randn(D, generator=g, device=DEV)
    return w_kd, w_ku, gamma


def _acts(seed, shape):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)


@pytest.mark.parametrize("N", [1, 100, 300])
def test_compress(oracle, N):
    D, Dc = 256, 16
    w_kd, _, _ = _weights(9950 + N, D, Dc)
    x = _acts(9960 + N, (N, D))
    c = gw.gold_compress(x, w_kd)
    torch.cuda.synchronize()
    assert rel_err(c, oracle.gold_compress(f64(x), f64(w_kd))) <= TOL_BF16


@pytest.mark.parametrize("N,gamma", [(1, True), (300, True), (129, False)])
def test_decompress(oracle, N, gamma):
    D, Dc = 256, 16
    _, w_ku, g = _weights(9970 + N, D, Dc)
    g = g if gamma else None
    x0, c = _acts(9980 + N, (N, D)), _acts(9990 + N, (N, Dc))
    kd = gw.gold_decompress(x0, c, w_ku, g, 1e-6)
    torch.cuda.synchronize()
    want = oracle.gold_decompress(f64(x0), f64(c), f64(w_ku), None if g is None else f64(g), 1e-6)
    assert rel_err(kd, want) <= TOL_BF16


def test_compress_then_decompress(oracle):
    """The cache entry the GPU wrote (bf16) feeds the decompression, as a GOLD layer reads it."""
    B, T, D, Dc = 2, 200, 512, 32
    w_kd, w_ku, g = _weights(10000, D, Dc)
    x, x0 = _acts(10001, (B, T, D)), _acts(10002, (B, T, D))
    c = gw.gold_compress(x, w_kd)
    kd = gw.gold_decompress(x0, c, w_ku, g, 1e-5)
    torch.cuda.synchronize()
    assert rel_err(c, oracle.gold_compress(f64(x), f64(w_kd))) <= TOL_BF16
    want = oracle.gold_decompress(f64(x0), f64(c), f64(w_ku), f64(g), 1e-5)
    assert rel_err(kd, want) <= TOL_BF16


def test_1p5b_shape_sampled_rows(oracle):
    """D = 2048 (H32 x 64), Dc = 128, B8 x T4096 tokens on the GPU; 64 rows through the oracle."""
    B, T, D, Dc = 8, 4096, 2048, 128
    w_kd, w_ku, g = _weights(10010, D, Dc)
    x, x0 = _acts(10011, (B * T, D)), _acts(10012, (B * T, D))
    c = gw.gold_compress(x, w_kd)
    kd = gw.gold_decompress(x0, c, w_ku, g, 1e-6)
    torch.cuda.synchronize()
    rows = torch.linspace(0, B * T - 1, 64).long().to(DEV)
    assert rel_err(c[rows], oracle.gold_compress(f64(x[rows]), f64(w_kd))) <= TOL_BF16
    want = oracle.gold_decompress(f64(x0[rows]), f64(c[rows]), f64(w_ku), f64(g), 1e-6)
    assert rel_err(kd[rows], want) <= TOL_BF16


def test_gold_argument_checks():
    L = bd.load()
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    N, D, Dc = 64, 256, 16
    w_kd, w_ku, g = _weights(10020, D, Dc)
    x0, c = _acts(10021, (N, D)), _acts(10022, (N, Dc))
    kd = torch.full((N, D), 3.0, device=DEV).to(torch.bfloat16)
    ws = torch.empty(bd.load().gold_decompress_workspace_bytes(N, D, Dc), dtype=torch.uint8,
                     device=DEV)

    def dec(out, eps=1e-6, nbytes=None, d=D):
        return L.gold_decompress(vp(x0), vp(c), vp(w_ku), vp(g), eps, vp(out), N, d, Dc, vp(ws),
                                 ws.numel() if nbytes is None else nbytes, stream)

    assert dec(x0) == bd.WKV_ERR_INVALID_ARG                 # output on top of an input
    assert dec(kd, eps=0.0) == bd.WKV_ERR_INVALID_ARG
    assert dec(kd, nbytes=ws.numel() - 1) == bd.WKV_ERR_WORKSPACE
    assert dec(kd, d=252) == bd.WKV_ERR_UNSUPPORTED          # rows not 16-byte multiples
    torch.cuda.synchronize()
    assert bool((kd == 3.0).all())
    assert dec(kd) == bd.WKV_OK
    assert L.gold_compress(vp(x0), vp(w_kd), vp(c), 0, D, Dc, None, 0, stream) == bd.WKV_OK


@pytest.mark.parametrize("N,D,Dc", [(257, 1000, 40), (130, 4096, 256), (64, 136, 8)])
def test_odd_widths(oracle, N, D, Dc):
    """Widths that are not multiples of the GEMM's tiles: D = 1000 (a partial last column
    tile, a 4-CTA cluster for the fused RMSNorm), Dc = 40 and 8 (a partial k-block of c, a
    partial column tile of the compression), D = 4096 (wider than one cluster: the fp32
    product and a separate RMSNorm), ragged N."""
    w_kd, w_ku, g = _weights(10100 + D, D, Dc)
    x, x0 = _acts(10101 + D, (N, D)), _acts(10102 + D, (N, D))
    c = gw.gold_compress(x, w_kd)
    kd = gw.gold_decompress(x0, c, w_ku, g, 1e-6)
    torch.cuda.synchronize()
    assert rel_err(c, oracle.gold_compress(f64(x), f64(w_kd))) <= TOL_BF16
    want = oracle.gold_decompress(f64(x0), f64(c), f64(w_ku), f64(g), 1e-6)
    assert rel_err(kd, want) <= TOL_BF16


def test_gemm_wait_timeout_is_reported(monkeypatch):
    """A zero spin budget makes the GEMM's bounded waits expire: the workspace status word
    reports it once, and the next call (normal budget) is correct and reports nothing."""
    N, D, Dc = 300, 512, 32
    w_kd, w_ku, g = _weights(10200, D, Dc)
    x0, c = _acts(10201, (N, D)), _acts(10202, (N, Dc))
    ws = bd.new_workspace(bd.load().gold_decompress_workspace_bytes(N, D, Dc), DEV)
    monkeypatch.setenv("GOLDWKV_FAULT", "timeout0")
    gw.gold_decompress(x0, c, w_ku, g, 1e-6, workspace=ws)
    assert bd.workspace_status(ws) == bd.WKV_ERR_TIMEOUT
    monkeypatch.delenv("GOLDWKV_FAULT")
    kd = gw.gold_decompress(x0, c, w_ku, g, 1e-6, workspace=ws)
    assert bd.workspace_status(ws) == bd.WKV_OK
    kd2 = gw.gold_decompress(x0, c, w_ku, g, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(kd, kd2)
