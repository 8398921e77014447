"""Thin ctypes binding of libgoldwkv (include/goldwkv.h): argument marshalling only.

Every step of the recurrence runs in the library's CUDA kernels; this module checks
tensor placement / dtype / contiguity, allocates outputs and workspace with torch on the
tensors' device, passes raw device pointers and the current CUDA stream, and turns a
non-OK status into an exception.  There is no CPU fallback: if the library is missing or
was not built, every call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libgoldwkv.so"

WKV_OK, WKV_ERR_INVALID_ARG, WKV_ERR_UNSUPPORTED, WKV_ERR_CUDA, WKV_ERR_TIMEOUT, WKV_ERR_WORKSPACE = range(6)
WKV_F32, WKV_BF16 = 0, 1
ALGOS = {"auto": 0, "recurrent": 1, "chunked": 2, "chunked_levels": 3}
HEAD_SIZE = 64

_lib = None


class WkvError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn}: {message} (status {status})")
        self.status = status


class _LN(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("eps", ctypes.c_float)]


class _GN(ctypes.Structure):
    _fields_ = [("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("eps", ctypes.c_float),
                ("gate", ctypes.c_void_p)]


def load(path: Path | str | None = None):
    """Load libgoldwkv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = Path(path) if path is not None else LIB_PATH
    if not p.exists():
        raise RuntimeError(
            f"{p} not found: build it with `python -m linear_attention_rnn_finch_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(str(p))
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.wkv6_prefill_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    L.wkv6_prefill_workspace_bytes.restype = sz
    L.wkv6_decode_workspace_bytes.argtypes = [i, i, i, i, i]
    L.wkv6_decode_workspace_bytes.restype = sz
    L.wkv6_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp, sz, vp]
    L.wkv6_prefill.restype = i
    L.wkv6_prefill_algo.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp, sz, vp]
    L.wkv6_prefill_algo.restype = i
    L.wkv6_prefill_static.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp]
    L.wkv6_prefill_static.restype = i
    L.wkv6_prefill_static_status.argtypes = [vp]
    L.wkv6_prefill_static_status.restype = i
    L.wkv6_segment_summary_workspace_bytes.argtypes = [i, i, i, i]
    L.wkv6_segment_summary_workspace_bytes.restype = sz
    L.wkv6_segment_summary.argtypes = [vp, vp, vp, i, vp, vp, i, i, i, i, i, vp, sz, vp]
    L.wkv6_segment_summary.restype = i
    L.wkv6_segment_carry.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
    L.wkv6_segment_carry.restype = i
    L.wkv6c2_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp, sz, vp]
    L.wkv6c2_prefill.restype = i
    L.wkv6c2_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp]
    L.wkv6c2_decode_step.restype = i
    L.wkv6_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp]
    L.wkv6_decode_step.restype = i
    L.wkv6_prefill_gn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp, sz, vp]
    L.wkv6_prefill_gn.restype = i
    L.wkv6_decode_step_gn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp]
    L.wkv6_decode_step_gn.restype = i
    L.wkv6_backward_workspace_bytes.argtypes = [i, i, i, i, i]
    L.wkv6_backward_workspace_bytes.restype = sz
    L.wkv6_backward.argtypes = [vp] * 14 + [i, i, i, i, i, vp, sz, vp]
    L.wkv6_backward.restype = i
    L.wkv6c2_backward_workspace_bytes.argtypes = [i, i, i, i, i]
    L.wkv6c2_backward_workspace_bytes.restype = sz
    L.wkv6c2_backward.argtypes = [vp] * 13 + [i, i, i, i, i, vp, sz, vp]
    L.wkv6c2_backward.restype = i
    L.gold_compress_workspace_bytes.argtypes = [ctypes.c_long, i, i]
    L.gold_compress_workspace_bytes.restype = sz
    L.gold_decompress_workspace_bytes.argtypes = [ctypes.c_long, i, i]
    L.gold_decompress_workspace_bytes.restype = sz
    L.gold_compress.argtypes = [vp, vp, vp, ctypes.c_long, i, i, vp, sz, vp]
    L.gold_compress.restype = i
    L.gold_decompress.argtypes = [vp, vp, vp, vp, ctypes.c_float, vp, ctypes.c_long, i, i, vp, sz, vp]
    L.gold_decompress.restype = i
    L.wkv6_workspace_status.argtypes = [vp, vp]
    L.wkv6_workspace_status.restype = i
    L.wkv6_status_string.argtypes = [i]
    L.wkv6_status_string.restype = ctypes.c_char_p
    L.wkv6_abi_version.argtypes = []
    L.wkv6_abi_version.restype = i
    if path is None:
        _lib = L
    return L


def status_string(status: int) -> str:
    return load().wkv6_status_string(status).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io(dtype) -> int:
    if dtype == torch.float32:
        return WKV_F32
    if dtype == torch.bfloat16:
        return WKV_BF16
    raise ValueError(f"unsupported I/O dtype {dtype}; expected float32 or bfloat16")


def _check(name, t, device, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_ptr(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ln_struct(ln, H, D, device):
    if ln is None:
        return None, None
    gamma, beta, eps = ln
    _check("ln.gamma", gamma, device, torch.float32, (H * D,))
    _check("ln.beta", beta, device, torch.float32, (H * D,))
    s = _LN(gamma.data_ptr(), beta.data_ptr(), float(eps))
    return s, ctypes.byref(s)


def _raise(fn, status):
    if status != WKV_OK:
        raise WkvError(fn, status, status_string(status))


def prefill_workspace_bytes(B, T, H, D, io_dtype, with_ln, algo="auto") -> int:
    return int(load().wkv6_prefill_workspace_bytes(B, T, H, D, _io(io_dtype), int(bool(with_ln)),
                                                   ALGOS[algo]))


def decode_workspace_bytes(B, H, D, io_dtype, with_ln) -> int:
    return int(load().wkv6_decode_workspace_bytes(B, H, D, _io(io_dtype), int(bool(with_ln))))


def wkv6_prefill(r, k, v, omega, u, state_in=None, *, ln=None, algo="auto", y=None,
                 state_out=None, want_state=True, workspace=None, stream=None):
    """Prefill over [B, T, H, D] inputs (fp32 or bf16), fp32 u [H, D] and optional fp32
    state_in [B, H, D, D].  ``ln`` = (gamma, beta, eps) applies LayerNorm over H*D.

    Returns (y, state_out); state_out is None when ``want_state`` is False and no
    ``state_out`` tensor was given.  ``state_out`` may be ``state_in`` (in-place update).
    """
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, dt, (B, T, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    if state_in is not None:
        _check("state_in", state_in, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, T, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, T, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check("state_out", state_out, dev, torch.float32, (B, H, D, D))
    ln_s, ln_p = _ln_struct(ln, H, D, dev)
    need = int(L.wkv6_prefill_workspace_bytes(B, T, H, D, _io(dt), int(ln is not None), ALGOS[algo]))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_prefill_algo(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state_in),
                                 _ptr(state_out), _ptr(y), B, T, H, D, _io(dt), ln_p, ALGOS[algo],
                                 _ptr(workspace), ws_bytes, _stream_ptr(dev, stream))
    del ln_s
    _raise("wkv6_prefill", st)
    return y, state_out


STATIC_SCRATCH_BYTES = 8 << 20   # WKV6_STATIC_SCRATCH_BYTES


def wkv6_prefill_static(r, k, v, omega, u, state_in=None, *, ln=None, y=None, state_out=None,
                        want_state=True, stream=None):
    """wkv6_prefill without a workspace: the library serves it from its built-in scratch
    (include/goldwkv.h, wkv6_prefill_static).  The library allocates nothing; this wrapper
    still allocates y / state_out with torch when they are not given.  Calls that may
    overlap in time on one device race on the shared scratch."""
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, dt, (B, T, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    if state_in is not None:
        _check("state_in", state_in, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, T, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, T, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check("state_out", state_out, dev, torch.float32, (B, H, D, D))
    ln_s, ln_p = _ln_struct(ln, H, D, dev)
    with torch.cuda.device(dev):
        st = L.wkv6_prefill_static(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state_in),
                                   _ptr(state_out), _ptr(y), B, T, H, D, _io(dt), ln_p,
                                   _stream_ptr(dev, stream))
    del ln_s
    _raise("wkv6_prefill_static", st)
    return y, state_out


def prefill_static_status(device=None, stream=None) -> int:
    """Synchronise the stream and read (then clear) the timeout record of the built-in
    scratch of ``device`` (include/goldwkv.h, wkv6_prefill_static_status): WKV_OK, or
    WKV_ERR_TIMEOUT if a bounded wait of a wkv6_prefill_static call expired since the last
    query (that call's outputs are undefined)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(load().wkv6_prefill_static_status(_stream_ptr(dev, stream)))


def segment_summary(k, v, omega, *, c2=False, workspace=None, stream=None):
    """State that k, v, omega [B, T, H, D] bf16 (T a multiple of 64) build from a zero state,
    [B, H, D, D] fp32, and each channel's total log2 decay over them, [B, H, D] fp32
    (include/goldwkv.h, wkv6_segment_summary)."""
    L = load()
    if k.dim() != 4:
        raise ValueError("k must be [B, T, H, D]")
    B, T, H, D = k.shape
    dev = k.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, torch.bfloat16, (B, T, H, D))
    s_loc = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    g = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    need = int(L.wkv6_segment_summary_workspace_bytes(B, T, H, D))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_segment_summary(_ptr(k), _ptr(v), _ptr(omega), int(bool(c2)), _ptr(s_loc),
                                    _ptr(g), B, T, H, D, WKV_BF16, _ptr(workspace), ws_bytes,
                                    _stream_ptr(dev, stream))
    _raise("wkv6_segment_summary", st)
    return s_loc, g


def segment_carry(s_loc, log2_decay, state0=None, *, stream=None):
    """States entering P segments from their summaries stacked segment-major, s_loc
    [P, B, H, D, D] and log2_decay [P, B, H, D]: returns [P + 1, B, H, D, D], entry p the
    state entering segment p and entry P the final state (include/goldwkv.h,
    wkv6_segment_carry)."""
    L = load()
    P, B, H, D, _ = s_loc.shape
    dev = s_loc.device
    _check("s_loc", s_loc, dev, torch.float32, (P, B, H, D, D))
    _check("log2_decay", log2_decay, dev, torch.float32, (P, B, H, D))
    if state0 is not None:
        _check("state0", state0, dev, torch.float32, (B, H, D, D))
    s_in = torch.empty((P + 1, B, H, D, D), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = L.wkv6_segment_carry(_ptr(state0), _ptr(s_loc), _ptr(log2_decay), _ptr(s_in), P, B,
                                  H, D, _stream_ptr(dev, stream))
    _raise("wkv6_segment_carry", st)
    return s_in


def wkv6c2_prefill(r, k, v, omega, uprime, state_in=None, *, ln=None, y=None, state_out=None,
                   want_state=True, workspace=None, stream=None):
    """Finch-C2 exact form (include/goldwkv.h, wkv6c2_prefill): the key is normalised by
    1 - w inside the library and the second value ``uprime`` [B, T, H, D] (dtype of r) is
    added to the readout in place of the static bonus.  Returns (y, state_out)."""
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega), ("uprime", uprime)):
        _check(name, t, dev, dt, (B, T, H, D))
    if state_in is not None:
        _check("state_in", state_in, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, T, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, T, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check("state_out", state_out, dev, torch.float32, (B, H, D, D))
    ln_s, ln_p = _ln_struct(ln, H, D, dev)
    need = int(L.wkv6_prefill_workspace_bytes(B, T, H, D, _io(dt), int(ln is not None), 0))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6c2_prefill(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(uprime), _ptr(state_in),
                              _ptr(state_out), _ptr(y), B, T, H, D, _io(dt), ln_p, _ptr(workspace),
                              ws_bytes, _stream_ptr(dev, stream))
    del ln_s
    _raise("wkv6c2_prefill", st)
    return y, state_out


def wkv6c2_decode_step(r, k, v, omega, uprime, state, *, ln=None, y=None, workspace=None,
                       stream=None):
    """Finch-C2 step over [B, H, D] inputs with second value ``uprime`` [B, H, D]; ``state``
    is updated in place.  Returns y."""
    L = load()
    if r.dim() != 3:
        raise ValueError("r must be [B, H, D]")
    B, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega), ("uprime", uprime)):
        _check(name, t, dev, dt, (B, H, D))
    _check("state", state, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, H, D))
    ln_s, ln_p = _ln_struct(ln, H, D, dev)
    need = int(L.wkv6_decode_workspace_bytes(B, H, D, _io(dt), int(ln is not None)))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)   # zero: LayerNorm row counters
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6c2_decode_step(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(uprime), _ptr(state),
                                  _ptr(y), B, H, D, _io(dt), ln_p, _ptr(workspace), ws_bytes,
                                  _stream_ptr(dev, stream))
    del ln_s
    _raise("wkv6c2_decode_step", st)
    return y


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Zero-filled device workspace (its leading status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and read (then clear) the workspace's device status word:
    WKV_OK, or WKV_ERR_TIMEOUT if a bounded wait in the chunked kernel expired."""
    dev = workspace.device
    with torch.cuda.device(dev):
        return int(load().wkv6_workspace_status(_ptr(workspace), _stream_ptr(dev, stream)))


def wkv6_decode_step(r, k, v, omega, u, state, *, ln=None, y=None, workspace=None, stream=None):
    """One step over [B, H, D] inputs; ``state`` [B, H, D, D] fp32 is updated in place.
    Returns y [B, H, D]."""
    L = load()
    if r.dim() != 3:
        raise ValueError("r must be [B, H, D]")
    B, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, dt, (B, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    _check("state", state, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, H, D))
    ln_s, ln_p = _ln_struct(ln, H, D, dev)
    need = int(L.wkv6_decode_workspace_bytes(B, H, D, _io(dt), int(ln is not None)))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)   # zero: LayerNorm row counters
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_decode_step(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state),
                                _ptr(y), B, H, D, _io(dt), ln_p, _ptr(workspace), ws_bytes,
                                _stream_ptr(dev, stream))
    del ln_s
    _raise("wkv6_decode_step", st)
    return y


def _gn_struct(gn, H, D, device, dtype, gate_shape):
    gamma, beta, eps, gate = gn
    _check("gn.gamma", gamma, device, torch.float32, (H * D,))
    _check("gn.beta", beta, device, torch.float32, (H * D,))
    if gate is not None:
        _check("gn.gate", gate, device, dtype, gate_shape)
    s = _GN(gamma.data_ptr(), beta.data_ptr(), float(eps),
            None if gate is None else gate.data_ptr())
    return s, ctypes.byref(s)


def wkv6_prefill_gn(r, k, v, omega, u, state_in=None, *, gn, y=None, state_out=None,
                    want_state=True, workspace=None, stream=None):
    """Base Finch prefill with its per-head GroupNorm and output gate (include/goldwkv.h,
    wkv6_prefill_gn).  ``gn`` = (gamma [H*D], beta [H*D], eps, gate [B, T, H, D] or None).
    Returns (y, state_out)."""
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, dt, (B, T, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    if state_in is not None:
        _check("state_in", state_in, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, T, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, T, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    if state_out is not None:
        _check("state_out", state_out, dev, torch.float32, (B, H, D, D))
    gn_s, gn_p = _gn_struct(gn, H, D, dev, dt, (B, T, H, D))
    need = int(L.wkv6_prefill_workspace_bytes(B, T, H, D, _io(dt), 1, 0))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_prefill_gn(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state_in),
                               _ptr(state_out), _ptr(y), B, T, H, D, _io(dt), gn_p,
                               _ptr(workspace), ws_bytes, _stream_ptr(dev, stream))
    del gn_s
    _raise("wkv6_prefill_gn", st)
    return y, state_out


def wkv6_decode_step_gn(r, k, v, omega, u, state, *, gn, y=None, workspace=None, stream=None):
    """Base Finch step with per-head GroupNorm and gate; ``gn`` = (gamma, beta, eps,
    gate [B, H, D] or None).  ``state`` is updated in place.  Returns y."""
    L = load()
    if r.dim() != 3:
        raise ValueError("r must be [B, H, D]")
    B, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega)):
        _check(name, t, dev, dt, (B, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    _check("state", state, dev, torch.float32, (B, H, D, D))
    if y is None:
        y = torch.empty((B, H, D), dtype=dt, device=dev)
    _check("y", y, dev, dt, (B, H, D))
    gn_s, gn_p = _gn_struct(gn, H, D, dev, dt, (B, H, D))
    # the GroupNorm stage runs inside the decode kernel: no workspace
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_decode_step_gn(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state),
                                   _ptr(y), B, H, D, _io(dt), gn_p, _ptr(workspace), ws_bytes,
                                   _stream_ptr(dev, stream))
    del gn_s
    _raise("wkv6_decode_step_gn", st)
    return y


def wkv6_backward(r, k, v, omega, u, state_in, dy, dstate_out=None, *, want_dstate_in=True,
                  workspace=None, stream=None):
    """Gradients of wkv6_prefill (no LayerNorm) given dy [B, T, H, D] (dtype of r) and the
    final-state gradient dstate_out [B, H, D, D] fp32 (None: zero).  Returns
    (dr, dk, dv, domega, du [H, D] fp32, dstate_in [B, H, D, D] fp32 or None)."""
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega), ("dy", dy)):
        _check(name, t, dev, dt, (B, T, H, D))
    _check("u", u, dev, torch.float32, (H, D))
    for name, t in (("state_in", state_in), ("dstate_out", dstate_out)):
        if t is not None:
            _check(name, t, dev, torch.float32, (B, H, D, D))
    dr, dk, dv, dom = (torch.empty((B, T, H, D), dtype=dt, device=dev) for _ in range(4))
    du = torch.empty((H, D), dtype=torch.float32, device=dev)
    ds_in = torch.empty((B, H, D, D), dtype=torch.float32, device=dev) if want_dstate_in else None
    need = int(L.wkv6_backward_workspace_bytes(B, T, H, D, _io(dt)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6_backward(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(u), _ptr(state_in),
                             _ptr(dy), _ptr(dstate_out), _ptr(dr), _ptr(dk), _ptr(dv), _ptr(dom),
                             _ptr(du), _ptr(ds_in), B, T, H, D, _io(dt), _ptr(workspace),
                             ws_bytes, _stream_ptr(dev, stream))
    _raise("wkv6_backward", st)
    return dr, dk, dv, dom, du, ds_in


def backward_workspace_bytes(B, T, H, D, io_dtype, c2=False) -> int:
    """Bytes of workspace wkv6_backward (or, c2, wkv6c2_backward) needs for these sizes."""
    L = load()
    fn = L.wkv6c2_backward_workspace_bytes if c2 else L.wkv6_backward_workspace_bytes
    return int(fn(B, T, H, D, _io(io_dtype)))


def gold_compress(x, w_kd, *, c=None, workspace=None, stream=None):
    """GOLD compression c = x W_KD (include/goldwkv.h): x [..., D] bf16, w_kd [Dc, D] bf16
    (the rows of the map).  Returns c [..., Dc] bf16."""
    L = load()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    D, Dc = x.shape[-1], w_kd.shape[0]
    N = x.numel() // D if D else 0
    _check("x", x, dev, torch.bfloat16)
    _check("w_kd", w_kd, dev, torch.bfloat16, (Dc, D))
    if c is None:
        c = torch.empty((*x.shape[:-1], Dc), dtype=torch.bfloat16, device=dev)
    _check("c", c, dev, torch.bfloat16, (*x.shape[:-1], Dc))
    need = int(L.gold_compress_workspace_bytes(N, D, Dc))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)   # zero: status word
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.gold_compress(_ptr(x), _ptr(w_kd), _ptr(c), N, D, Dc, _ptr(workspace), ws_bytes,
                             _stream_ptr(dev, stream))
    _raise("gold_compress", st)
    return c


def gold_decompress(x0, c, w_ku, gamma=None, eps=1e-6, *, kd=None, workspace=None, stream=None):
    """TokenCat decompression RMSNorm(concat(x0, c) W_KU) (include/goldwkv.h): x0 [..., D]
    and c [..., Dc] bf16, w_ku [D, D + Dc] bf16 (the rows of the map), gamma [D] fp32 or
    None.  Returns kd [..., D] bf16."""
    L = load()
    dev = x0.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    D, Dc = x0.shape[-1], c.shape[-1]
    N = x0.numel() // D if D else 0
    _check("x0", x0, dev, torch.bfloat16)
    _check("c", c, dev, torch.bfloat16, (*x0.shape[:-1], Dc))
    _check("w_ku", w_ku, dev, torch.bfloat16, (D, D + Dc))
    if gamma is not None:
        _check("gamma", gamma, dev, torch.float32, (D,))
    if kd is None:
        kd = torch.empty_like(x0)
    _check("kd", kd, dev, torch.bfloat16, tuple(x0.shape))
    need = int(L.gold_decompress_workspace_bytes(N, D, Dc))
    if workspace is None and need > 0:
        workspace = new_workspace(need, dev)   # zero: status word
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.gold_decompress(_ptr(x0), _ptr(c), _ptr(w_ku), _ptr(gamma), float(eps), _ptr(kd),
                               N, D, Dc, _ptr(workspace), ws_bytes, _stream_ptr(dev, stream))
    _raise("gold_decompress", st)
    return kd


def wkv6c2_backward(r, k, v, omega, state_in, dy, dstate_out=None, *, want_dstate_in=True,
                    want_duprime=True, workspace=None, stream=None):
    """Gradients of wkv6c2_prefill (no LayerNorm) for dy [B, T, H, D] and dstate_out
    [B, H, D, D] fp32 (None: zero).  Returns (dr, dk, dv, domega, duprime or None,
    dstate_in or None)."""
    L = load()
    if r.dim() != 4:
        raise ValueError("r must be [B, T, H, D]")
    B, T, H, D = r.shape
    dev, dt = r.device, r.dtype
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (no CPU implementation)")
    for name, t in (("r", r), ("k", k), ("v", v), ("omega", omega), ("dy", dy)):
        _check(name, t, dev, dt, (B, T, H, D))
    for name, t in (("state_in", state_in), ("dstate_out", dstate_out)):
        if t is not None:
            _check(name, t, dev, torch.float32, (B, H, D, D))
    dr, dk, dv, dom = (torch.empty((B, T, H, D), dtype=dt, device=dev) for _ in range(4))
    dup = torch.empty((B, T, H, D), dtype=dt, device=dev) if want_duprime else None
    ds_in = torch.empty((B, H, D, D), dtype=torch.float32, device=dev) if want_dstate_in else None
    need = int(L.wkv6c2_backward_workspace_bytes(B, T, H, D, _io(dt)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = L.wkv6c2_backward(_ptr(r), _ptr(k), _ptr(v), _ptr(omega), _ptr(state_in), _ptr(dy),
                               _ptr(dstate_out), _ptr(dr), _ptr(dk), _ptr(dv), _ptr(dom),
                               _ptr(dup), _ptr(ds_in), B, T, H, D, _io(dt), _ptr(workspace),
                               ws_bytes, _stream_ptr(dev, stream))
    _raise("wkv6c2_backward", st)
    return dr, dk, dv, dom, dup, ds_in
