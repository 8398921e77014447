#!/usr/bin/env python3
"""Benchmark of the WKV6 hot path on B200: prefill tokens/s (+ decode GB/s), one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step): one wkv6_prefill call over the 1.5B-class layer shape,
B=8, T=4096, H=32, D=64, bf16 r/k/v/omega/y, fp32 u and state, initial state ~N(0,0.1)
(seeded synthetic data).  The inputs (537 MB) exceed the 126 MB L2, so no flush is needed
between timed steps.  For N > 1 (torchrun, one rank per GPU) every rank runs its own
independent batch of that shape (weak scaling; the path has no collective) and `value` is
all tokens of all ranks over the slowest rank's device time.

The line also reports: the dominant kernel's roofline fraction (algorithmic bytes per
launch / CUDA-event launch time vs. the measured HBM copy bandwidth), SM clocks sampled
with nvidia-smi during the timed region, an end-to-end figure through the public API with
host buffers (pinned host -> device inputs, prefill, device -> host y and state inside the
timed region) and the fp64 oracle timed on the host cores on a bounded sample.
The other measurements go, one short record each, into the list `more` (workload with its
sizes, ms per call, value and unit, roofline bound and fraction, and for decode also the
fraction from the DRAM bytes ncu counted): the decode step, the long-context and
decay-extreme (+ LayerNorm) prefill shapes, the 1.5B layer in Finch-C2's form and with base
Finch's GroupNorm + gate, the backward of both forms (FP32 CUDA-core roofline), and GOLD
compression + decompression (bf16 tensor roofline).  `--only backward|backward_c2|gold`
prints one of those alone, in full.  Every API call in a timed loop sits in an NVTX range
named after the entry point.

`--impl reference` times the oracle (the only reference implementation of this path) on the
host cores on the same workload, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from linear_attention_rnn_finch_b200 import workloads as W  # noqa: E402

METRIC = "WKV prefill tokens/s (H=32, D=64) and decode GB/s; fraction of roofline"
PREFILL_CFG = W.CONFIGS[1]
DECODE_CFG = W.CONFIGS[3]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0   # an earlier dense bf16 GEMM measurement on B200 (burst)


def prefill_bytes(B, T, H, D=64, esz=2):
    """Algorithmic HBM bytes of one prefill launch: r, k, v, omega in, y out (per
    token-head 5*D*esz), fp32 state in and out (2*D*D*4 per head), u."""
    return 5 * D * esz * B * T * H + 2 * D * D * 4 * B * H + H * D * 4


def backward_flops(B, T, H, D=64):
    """Algorithmic fp32 FLOPs of one backward call: three scans over every (b,h), each per
    token a readout (D*D fused multiply-adds) and a state update w*X + a*b (D*D multiplies
    and D*D fused multiply-adds): 2 + 1 + 2 = 5 FLOPs per state entry per scan."""
    return 3 * 5 * D * D * B * T * H


def backward_bytes(B, T, H, D=64, esz=2):
    """Algorithmic HBM bytes of one backward call: r, k, v, omega, dy in and dr, dk, dv,
    domega out (9*D*esz per token-head), state_in and dS_T in, dS_0 out (3*D*D*4 per head)."""
    return 9 * D * esz * B * T * H + 3 * D * D * 4 * B * H + 2 * H * D * 4


# FP32 CUDA-core peak of a B200 from its unit counts and clock: 148 SMs x 128 FP32 lanes x
# 2 FLOPs per fused multiply-add x 1.965 GHz (clocks.max.sm).
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def decode_bytes(B, H, D=64, esz=2):
    """Algorithmic bytes of one decode step: state read + written, r/k/v/omega in, y out."""
    return B * H * (2 * D * D * 4 + 5 * D * esz) + H * D * 4


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of each dominant kernel, with the hash of the sources the captured build came
# from; reported only while the sources still hash to that value (else null).
CSRC = ROOT / "linear_attention_rnn_finch_b200" / "csrc"
NCU_TRAFFIC = {
    "prefill": {"sources": ("chunked_fast_sm100.cu", "chunk_tiles.cuh", "sm100_ptx.cuh", "common.cuh",
                            "internal.h"),
                "sha256_16": "e07ae25d1780988a", "bytes": 541190912 + 118802176,
                "workload": (8, 4096, 32)},
    "decode": {"sources": ("decode.cu", "common.cuh"),
               "sha256_16": "0468671fdbdebeab", "bytes": 138433024 + 78395392,
               "workload": (256, 32)},
}


def ncu_traffic(kind: str, workload: tuple):
    import hashlib
    rec = NCU_TRAFFIC[kind]
    h = hashlib.sha256()
    for name in rec["sources"]:
        h.update((CSRC / name).read_bytes())
    if h.hexdigest()[:16] != rec["sha256_16"] or tuple(workload) != rec["workload"]:
        return None
    return rec["bytes"]


def sig(x, digits=4):
    """x rounded to `digits` significant figures (keeps the printed line short)."""
    if x is None or x == 0 or not isinstance(x, float):
        return x
    from math import floor, log10
    return round(x, max(0, digits - 1 - int(floor(log10(abs(x))))))


def compact(line: dict) -> dict:
    """One secondary measurement as a short record: workload, ms per call, value and unit,
    the roofline bound and fraction, and (where an ncu capture of the same sources exists)
    the fraction computed from the DRAM bytes ncu counted instead of the algorithmic ones."""
    r = line["roofline"]
    out = {"w": line["workload"], "ms": sig(line["ms_per_call"]),
           "v": sig(float(line["value"])), "u": line["unit"],
           "bound": r["bound"], "frac": sig(r["frac"], 3)}
    if r.get("dram_frac") is not None:
        out["dram_frac"] = sig(r["dram_frac"], 3)
    return out


def nvtx(name: str):
    """NVTX range around one API call (visible in an nsys or ncu timeline)."""
    return torch.cuda.nvtx.range(name)


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------------------ clock sampler
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = {}

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, name):
        self.marks[name] = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]),
                                 reasons={n: (v.strip() == "Active") for n, v in zip(self.REASONS, f[5:9])}))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for r in rows for n, a in r["reasons"].items() if a})
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------------ distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def other_prefill(cfg, dev, world, hbm, algo, steps, c2=False, gn=False):
    """Device-timed prefill calls of another workload shape: one line of its own (tokens/s and
    the fraction of the HBM roofline), inputs resident in HBM and larger than L2.  c2: the
    Finch-C2 entry point (normalised key, second value u' read in place of the bonus).  gn:
    base Finch's output stage (per-head GroupNorm, then a gate tensor read from HBM)."""
    import linear_attention_rnn_finch_b200 as gw
    inp = W.make_prefill_inputs(cfg, dev)
    g = torch.Generator(device=dev).manual_seed(cfg.seed + 5)
    if c2:
        inp["uprime"] = (torch.randn(inp["r"].shape, generator=g, device=dev) * 0.125).to(cfg.dtype)
    B, T, H, D = cfg.B, cfg.T, cfg.H, cfg.D
    if gn:
        gn_args = (1.0 + 0.1 * torch.randn(H * D, generator=g, device=dev),
                   0.1 * torch.randn(H * D, generator=g, device=dev), 64e-5,
                   (2.0 * torch.rand(inp["r"].shape, generator=g, device=dev)).to(cfg.dtype))
    ln = (inp["gamma"], inp["beta"], inp["eps"]) if cfg.ln else None
    ws = gw.new_workspace(gw.prefill_workspace_bytes(B, T, H, D, cfg.dtype, ln is not None or gn,
                                                     algo), dev)
    y = torch.empty_like(inp["r"])
    s_out = torch.empty_like(inp["state0"])
    args_p = [inp[n] for n in ("r", "k", "v", "omega")]

    def call():
        with nvtx("wkv6_prefill_gn" if gn else "wkv6c2_prefill" if c2 else "wkv6_prefill"):
            call_()

    def call_():
        if gn:
            gw.wkv6_prefill_gn(*args_p, inp["u"], inp["state0"], gn=gn_args, y=y, state_out=s_out,
                               workspace=ws)
        elif c2:
            gw.wkv6c2_prefill(*args_p, inp["uprime"], inp["state0"], ln=ln, y=y, state_out=s_out,
                              workspace=ws)
        else:
            gw.wkv6_prefill(*args_p, inp["u"], inp["state0"], ln=ln, y=y, state_out=s_out,
                            algo=algo, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    # + u' read (C2) or + gate read (GroupNorm)
    nbytes = prefill_bytes(B, T, H, D) + (B * T * H * D * 2 if c2 or gn else 0)
    # the roofline counts only the bytes the operation itself must move (LayerNorm's fp32
    # staging of y is not counted)
    nbytes_note = ("GroupNorm + gate runs in the recurrence kernels' output stage" if gn else
                   "LayerNorm runs inside the level kernel's launch on co-resident CTAs when the "
                   "recurrence's CTAs leave SMs free (else as a second pass) over an fp32 staging "
                   "of y, not counted in the algorithmic bytes" if cfg.ln else None)
    name = ("wkv6c2_" + cfg.name[5:]) if c2 else (cfg.name + "_groupnorm_gate") if gn else cfg.name
    form = ("Finch-C2 (normalised key, second value)" if c2 else
            "base Finch (static bonus), per-head GroupNorm and gate" if gn else
            "base Finch (static bonus)")
    line = {"workload": f"{name} B{B} T{T} H{H}", "B": B, "T": T, "H": H, "D": D, "io": "bf16",
            "form": form, "ln": bool(cfg.ln), "steps": steps, "ms_per_call": ms,
            "value": world * B * T / (ms / 1e3), "unit": "tokens/s",
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm,
                         "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm,
                         "algorithmic_bytes_per_call": nbytes}}
    if nbytes_note:
        line["note"] = nbytes_note
    del inp, y, s_out, ws
    if gn:
        del gn_args
    torch.cuda.empty_cache()
    return line


def backward_line(cfg, dev, world, steps, c2=False):
    """Device-timed wkv6_backward (or, c2, wkv6c2_backward) on the prefill workload's shape
    (bf16 I/O): gradients of every input for a random dy and final-state gradient."""
    import linear_attention_rnn_finch_b200 as gw
    inp = W.make_prefill_inputs(cfg, dev)
    g = torch.Generator(device=dev).manual_seed(cfg.seed + 7)
    dy = torch.randn(inp["r"].shape, generator=g, device=dev).to(cfg.dtype)
    dS = torch.randn(inp["state0"].shape, generator=g, device=dev) * 0.1
    B, T, H, D = cfg.B, cfg.T, cfg.H, cfg.D
    ws = torch.empty(gw.backward_workspace_bytes(B, T, H, D, cfg.dtype, c2=c2), dtype=torch.uint8,
                     device=dev)
    names = ("r", "k", "v", "omega", "state0") if c2 else ("r", "k", "v", "omega", "u", "state0")
    args_b = [inp[n] for n in names]

    def call():
        with nvtx("wkv6c2_backward" if c2 else "wkv6_backward"):
            if c2:
                return gw.wkv6c2_backward(*args_b, dy, dS, workspace=ws)
            return gw.wkv6_backward(*args_b, dy, dS, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    flops, nbytes = backward_flops(B, T, H, D), backward_bytes(B, T, H, D)
    # base form: 2 reversals + fast + level kernels for dv (+ 2 segment kernels when the
    # sequence is split), the tensor-core dr and dk readouts, the decay gradient's two
    # column-sum kernels and its scan, the dr and dk scans (which exit at once unless a
    # (b,h) fell back) and the du sum.
    # (Finch-C2: the same launches; its dv prefill forms the query k (1 - w) inside)
    launches_per_call = 12
    line = {"workload": ("wkv6c2_backward" if c2 else "wkv6_backward") + f" B{B} T{T} H{H}",
            "B": B, "T": T, "H": H, "D": D, "io": "bf16", "steps": steps, "ms_per_call": ms,
            "value": world * B * T / (ms / 1e3), "unit": "tokens/s",
            "roofline": {"bound": "alu", "achieved": flops / (ms / 1e3) / 1e12,
                         "peak": ALU_FP32_TFLOPS, "unit": "TFLOP/s",
                         "frac": flops / (ms / 1e3) / 1e12 / ALU_FP32_TFLOPS,
                         "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz",
                         "algorithmic_flops_per_call": flops},
            "hbm": {"achieved_gbs": nbytes / (ms / 1e3) / 1e9, "algorithmic_bytes_per_call": nbytes},
            "gpu_launches": launches_per_call * steps,
            "kernels": ("dr and dk as chunked tensor-core readouts (wkv6_bwd_readout_tc_kernel "
                        "x2, kn = k (1 - w) formed in the dr pass), the decay gradient from "
                        "their pair terms and kn's direct term, dv through the chunked prefill "
                        "on time-reversed copies with the query k (1 - w) formed inside; the "
                        "CUDA-core scans run only for a (b,h) that falls back") if c2 else
                       ("dr and dk as chunked tensor-core readouts of the forward and the "
                        "reversed state (wkv6_bwd_readout_tc_kernel x2), the decay gradient from "
                        "their pair terms (wkv6_bwd_col_sums_kernel x2, wkv6_bwd_domega_kernel), dv "
                        "through the chunked tensor-core prefill on time-reversed copies "
                        "(reverse_tokens_kernel x2, wkv6_fast_kernel, wkv6_chunked_kernel); the "
                        "CUDA-core scans run only for a (b,h) whose decays the one-sided factors "
                        "cannot take"),
            "note": "algorithmic FLOPs are the three recurrences (dr, dk, dv) at 5 FLOPs per "
                    "state entry per token; dr, dk and dv run on the tensor cores, on three "
                    "streams forked from and joined to the caller's"}
    del inp, dy, dS, ws, args_b
    torch.cuda.empty_cache()
    return line


def gold_line(dev, world, steps, B=8, T=4096, D=2048, Dc=128):
    """Device-timed GOLD compression + TokenCat decompression of every token of the 1.5B-layer
    shape (D = H*64 = 2048, Dc = D/16): one step = gold_compress then gold_decompress."""
    import linear_attention_rnn_finch_b200 as gw
    N = B * T
    g = torch.Generator(device=dev).manual_seed(1005)
    x = torch.randn((N, D), generator=g, device=dev).to(torch.bfloat16)
    x0 = torch.randn((N, D), generator=g, device=dev).to(torch.bfloat16)
    w_kd = (torch.randn((Dc, D), generator=g, device=dev) / D ** 0.5).to(torch.bfloat16)
    w_ku = (torch.randn((D, D + Dc), generator=g, device=dev) / (D + Dc) ** 0.5).to(torch.bfloat16)
    gamma = 1.0 + 0.1 * torch.randn(D, generator=g, device=dev)
    c = torch.empty((N, Dc), dtype=torch.bfloat16, device=dev)
    kd = torch.empty_like(x0)
    L = gw.load()
    ws_c = gw.new_workspace(L.gold_compress_workspace_bytes(N, D, Dc), dev)
    ws_d = gw.new_workspace(L.gold_decompress_workspace_bytes(N, D, Dc), dev)

    def call():
        with nvtx("gold_compress"):
            gw.gold_compress(x, w_kd, c=c, workspace=ws_c)
        with nvtx("gold_decompress"):
            gw.gold_decompress(x0, c, w_ku, gamma, 1e-6, kd=kd, workspace=ws_d)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    flops = 2 * N * D * Dc + 2 * N * (D + Dc) * D
    peak = bf16_peak()
    line = {"workload": f"gold_compress_decompress N{N} D{D} Dc{Dc}", "N_tokens": N, "D": D,
            "Dc": Dc, "io": "bf16", "steps": steps, "ms_per_call": ms,
            "value": world * N / (ms / 1e3), "unit": "tokens/s",
            "roofline": {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": flops / (ms / 1e3) / 1e12 / peak,
                         "peak_source": "measured bf16_tflops (cuBLAS burst)",
                         "algorithmic_flops_per_call": flops},
            "gpu_launches": 2 * steps,
            "note": "gold_gemm_kernel (tcgen05) twice per step: the compression, then the "
                    "decompression with RMSNorm in its epilogue"}
    del x, x0, w_kd, w_ku, gamma, c, kd, ws_c, ws_d
    torch.cuda.empty_cache()
    return line


def seqpar_line(dev, world, rank, steps, hbm):
    """The long-context shape (B1 T262144 H64) as ONE sequence split across the ranks
    (linear_attention_rnn_finch_b200/seqpar.py): rank p holds tokens p*T/N .. (p+1)*T/N - 1;
    per call: the span's summary, one all-gather of the summaries (NCCL), the carry, the
    span's prefill.  Time is the slowest rank's (strong scaling: the work is fixed)."""
    import torch.distributed as dist
    import linear_attention_rnn_finch_b200 as gw
    from linear_attention_rnn_finch_b200 import seqpar
    cfg = W.CONFIGS[2]
    B, T, H, D = cfg.B, cfg.T, cfg.H, cfg.D
    if T % (64 * world):
        raise ValueError("the sequence must split into chunk-aligned spans")
    tp = T // world
    full = W.make_prefill_inputs(cfg, dev)
    a = [full[n][:, rank * tp:(rank + 1) * tp].contiguous() for n in ("r", "k", "v", "omega")]
    u, s0 = full["u"], full["state0"]
    del full
    torch.cuda.empty_cache()

    def call():
        with nvtx("seqpar_prefill"):
            return seqpar.prefill_sequence_parallel(*a, u, s0)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    dist.barrier()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    nbytes = prefill_bytes(B, T, H, D)
    return {"workload": f"wkv6_prefill_long_ctx B{B} T{T} H{H} split over {world} rank(s)",
            "ms_per_call": ms, "value": B * T / (ms / 1e3), "unit": "tokens/s",
            "roofline": {"bound": "hbm", "frac": nbytes / (ms / 1e3) / 1e9 / (hbm * world)},
            "note": "strong scaling of one sequence; frac against N GPUs' HBM bandwidth"}


def bf16_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        return float(json.loads(p.read_text())["bf16_tflops"])
    return FALLBACK_BF16_TFLOPS


# ------------------------------------------------------------------------------ oracle timing
def oracle_sample(cfg, b_rows: int, t_tokens: int, seed_offset: int = 0):
    """Inputs of the oracle's bounded sample: b_rows batch rows x t_tokens tokens of cfg,
    drawn by the same seeded generator on the host."""
    import numpy as np
    inp = W.make_prefill_inputs(cfg, "cpu", B=b_rows, T=t_tokens, seed=cfg.seed + seed_offset)
    a = [inp[n].to(torch.float64).numpy() for n in ("r", "k", "v", "omega")]
    return a, inp["u"].double().numpy(), inp["state0"].double().numpy(), np


def time_oracle(cfg, b_rows, t_tokens, reps=1):
    import oracle as oracle_pkg
    orc = oracle_pkg.get()
    a, u, s0, _ = oracle_sample(cfg, b_rows, t_tokens)
    nthreads = oracle_pkg.default_threads()
    best = None
    for _ in range(reps):
        t0 = time.perf_counter()
        orc.prefill(*a, u, s0, nthreads=nthreads)
        dt = time.perf_counter() - t0
        best = dt if best is None else min(best, dt)
    return b_rows * t_tokens / best, nthreads, best


def sized_sample(cfg, seconds: float):
    """(batch rows, tokens) of a sample of cfg that the oracle finishes in about `seconds`
    (at most the whole workload): grow a probe until it runs >= 0.5 s, then scale."""
    rows, t_tok = 1, 128
    while True:
        tps, _, secs = time_oracle(cfg, rows, t_tok)
        if secs >= 0.5 or (rows == cfg.B and t_tok == cfg.T):
            break
        if t_tok < cfg.T:
            t_tok = min(cfg.T, t_tok * 4)
        else:
            rows = min(cfg.B, rows * 2)
    tokens = max(64, int(tps * seconds))
    if tokens >= cfg.T:
        return max(1, min(cfg.B, tokens // cfg.T)), cfg.T
    return 1, tokens


# ------------------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    import linear_attention_rnn_finch_b200 as gw
    from linear_attention_rnn_finch_b200 import binding

    binding.load()
    dev = torch.device("cuda", local)
    cfg = PREFILL_CFG if args.batch is None else PREFILL_CFG.with_(B=args.batch)
    B, T, H, D = cfg.B, cfg.T, cfg.H, cfg.D
    inp = W.make_prefill_shard(cfg, dev, rank)
    ws = gw.new_workspace(gw.prefill_workspace_bytes(B, T, H, D, cfg.dtype, False, args.algo), dev)
    y = torch.empty_like(inp["r"])
    s_out = torch.empty_like(inp["state0"])
    stream = torch.cuda.current_stream(dev)
    args_p = [inp[n] for n in ("r", "k", "v", "omega")]
    algo = args.algo

    def step():
        with nvtx("wkv6_prefill"):
            gw.wkv6_prefill(*args_p, inp["u"], inp["state0"], y=y, state_out=s_out, algo=algo,
                            workspace=ws)

    sampler = ClockSampler(local)
    sampler.start()
    # untimed warm-up: W steps, then ~1 s of steps so clocks settle and the sampler sees load
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t_end = time.time() + (0.0 if args.no_clock_warm else 1.0)
    while time.time() < t_end:
        for _ in range(20):
            step()
        torch.cuda.synchronize()

    barrier(world)
    torch.cuda.synchronize()
    sampler.mark("t0")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        step()
        ev[i + 1].record(stream)
    ev[-1].synchronize()
    torch.cuda.synchronize()
    barrier(world)
    sampler.mark("t1")
    launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms_max = max_over_ranks(total_ms, world)
    tokens_all = sum_over_ranks(float(B * T * args.steps), world)
    value = tokens_all / (total_ms_max / 1e3)
    ms_per_step = total_ms_max / args.steps

    hbm, peak_kind = peaks()
    bytes_launch = prefill_bytes(B, T, H, D)
    avg_launch_ms = statistics.mean(launch_ms)
    achieved = bytes_launch / (avg_launch_ms / 1e3) / 1e9
    # the chunked path launches the fast kernel and the level kernel (which finishes any
    # sequence handed over to it); the fp32 recurrence is one kernel; no LayerNorm here
    chunked = algo == "chunked" or (algo == "auto" and cfg.dtype == torch.bfloat16)
    launches_per_step = 2 if chunked else 1

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "wkv6_prefill_1p5b_layer" + ("" if args.batch is None else f"_B{B}"),
                   "B": B, "T": T, "H": H, "D": D,
                   "io": "bf16", "state": "fp32", "algo": algo,
                   "parallelism": f"dp{world}, independent batches, no collective",
                   "l2": "inputs (537 MB) larger than L2, no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm,
                     "traffic": ncu_traffic("prefill", (B, T, H)) if chunked else None,
                     "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": bytes_launch,
                     "kernel": "wkv6_fast_kernel + wkv6_chunked_kernel, per call"},
        "gpu_launches": launches_per_step * args.steps,
    }
    more = []   # the other measurements, printed compactly under "more"

    # decode: 100 steps back to back, state in place; GB/s of algorithmic bytes
    if not args.no_decode:
        dcfg = DECODE_CFG
        dinp = W.make_decode_shard(dcfg, dev, rank)
        state = dinp["state0"].clone()
        ybuf = torch.empty_like(dinp["r"][0])
        dsteps = dcfg.steps
        dargs = [[dinp[n][s] for n in ("r", "k", "v", "omega")] for s in range(dsteps)]

        def dstep(s):
            with nvtx("wkv6_decode_step"):
                gw.wkv6_decode_step(*dargs[s], dinp["u"], state, y=ybuf)

        for s in range(dsteps):
            dstep(s)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(dsteps):
            dstep(s)
        e1.record(stream)
        e1.synchronize()
        barrier(world)
        dms = max_over_ranks(e0.elapsed_time(e1), world) / dsteps
        dbytes = decode_bytes(dcfg.B, dcfg.H, dcfg.D)
        dgbs = dbytes / (dms / 1e3) / 1e9
        # the same steps with Finch-C2's LayerNorm over each row's H*D outputs, fused into the
        # decode kernel (one launch per step; one zero-filled workspace for all steps)
        g = torch.Generator(device=dev).manual_seed(dcfg.seed + 3)
        lnp = (1.0 + 0.1 * torch.randn(dcfg.H * dcfg.D, generator=g, device=dev),
               0.1 * torch.randn(dcfg.H * dcfg.D, generator=g, device=dev), 1e-5)
        lnws = gw.new_workspace(gw.decode_workspace_bytes(dcfg.B, dcfg.H, dcfg.D, dcfg.dtype, True), dev)

        def dstep_ln(s):
            with nvtx("wkv6_decode_step"):
                gw.wkv6_decode_step(*dargs[s], dinp["u"], state, ln=lnp, y=ybuf, workspace=lnws)

        for s in range(dsteps):
            dstep_ln(s)
        torch.cuda.synchronize()
        barrier(world)
        e0.record(stream)
        for s in range(dsteps):
            dstep_ln(s)
        e1.record(stream)
        e1.synchronize()
        barrier(world)
        dms_ln = max_over_ranks(e0.elapsed_time(e1), world) / dsteps
        # + gamma and beta read once per step
        dbytes_ln = dbytes + 2 * dcfg.H * dcfg.D * 4
        dgbs_ln = dbytes_ln / (dms_ln / 1e3) / 1e9
        # DRAM-only rate: the bytes ncu counted at DRAM per step (part of the state round
        # trip is served from L2 between back-to-back steps) over the same time
        dtraffic = ncu_traffic("decode", (dcfg.B, dcfg.H))
        more.append({"workload": f"wkv6_decode_step B{dcfg.B} H{dcfg.H}", "ms_per_call": dms,
                     "value": dgbs * world, "unit": "GB/s",
                     "roofline": {"bound": "hbm", "frac": dgbs / hbm,
                                  "dram_frac": None if dtraffic is None else
                                  dtraffic / (dms / 1e3) / 1e9 / hbm}})
        more.append({"workload": f"wkv6_decode_step_layernorm B{dcfg.B} H{dcfg.H} (one kernel)",
                     "ms_per_call": dms_ln, "value": dgbs_ln * world, "unit": "GB/s",
                     "roofline": {"bound": "hbm", "frac": dgbs_ln / hbm}})

        del dinp, dargs, state, lnws

    # the other prefill shapes: long context (one sequence per head; the library splits it
    # into segments across SMs), the decay-extreme stress with LayerNorm, and the 1.5B layer
    # in Finch-C2's form and with base Finch's GroupNorm + gate
    if not args.no_other:
        more += [other_prefill(W.CONFIGS[2], dev, world, hbm, args.algo, steps=5),
                 other_prefill(W.CONFIGS[4], dev, world, hbm, args.algo, steps=5),
                 other_prefill(W.CONFIGS[1], dev, world, hbm, args.algo, steps=10, c2=True),
                 other_prefill(W.CONFIGS[1], dev, world, hbm, args.algo, steps=10, gn=True),
                 backward_line(W.CONFIGS[1], dev, world, steps=5),
                 backward_line(W.CONFIGS[1], dev, world, steps=5, c2=True),
                 gold_line(dev, world, steps=10)]
    if more:
        out["more"] = [compact(m) for m in more]

    # end to end through the public API with host buffers: every step copies its inputs in
    # from pinned host memory and reads y and the final state back.  Steps are pipelined over
    # two device buffer sets on three streams (copy in, compute, copy out), so the copy-in of
    # step i overlaps the copy-out of step i-1 (PCIe is full duplex).
    if not args.no_e2e:
        names = ("r", "k", "v", "omega", "u", "state0")
        host = {n: inp[n].cpu().pin_memory() for n in names}
        dbuf = [{n: torch.empty_like(inp[n]) for n in names} for _ in range(2)]
        ybuf = [torch.empty_like(y) for _ in range(2)]
        sbuf = [torch.empty_like(s_out) for _ in range(2)]
        wsb = [ws, gw.new_workspace(ws.numel(), dev)]
        y_h = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
        s_h = torch.empty(s_out.shape, dtype=s_out.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = y_h.numel() * y_h.element_size() + s_h.numel() * s_h.element_size()
        s_in, s_cmp, s_out_st = (torch.cuda.Stream(dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i & 1
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev_cmp[b])          # step i-2 has consumed this input set
                for n in names:
                    dbuf[b][n].copy_(host[n], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                if used[b]:
                    s_cmp.wait_event(ev_out[b])         # step i-2's outputs have been read back
                d = dbuf[b]
                gw.wkv6_prefill(d["r"], d["k"], d["v"], d["omega"], d["u"], d["state0"],
                                y=ybuf[b], state_out=sbuf[b], algo=algo, workspace=wsb[b],
                                stream=s_cmp)
                ev_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out_st):
                s_out_st.wait_event(ev_cmp[b])
                y_h.copy_(ybuf[b], non_blocking=True)
                s_h.copy_(sbuf[b], non_blocking=True)
                ev_out[b].record(s_out_st)
            used[b] = True

        e2e_steps = max(3, min(args.steps, 10))
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        s_in.wait_stream(s_out_st)
        e1.record(s_in)
        e1.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        etok = sum_over_ranks(float(B * T * e2e_steps), world)
        out["e2e"] = {"value": etok / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                      "note": "copy in / compute / copy out streams, 2 buffer sets"}
        del dbuf, ybuf, sbuf, wsb

    sampler.stop()
    out["clocks"] = sampler.summary(sampler.marks.get("t0", 0) - 1.0, sampler.marks.get("t1", 0))

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b_rows, t_tok = sized_sample(cfg, 12.0)
        tps, cores, secs = time_oracle(cfg, b_rows, t_tok)
        reps = 1
        while secs * reps < 8.0 and reps < 64:   # whole workload too quick: repeat it
            reps *= 2
        if reps > 1:
            tps, cores, secs1 = time_oracle(cfg, b_rows, t_tok, reps=reps)
            secs = secs1 * reps
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": f"{b_rows} rows x {t_tok} tokens x {H} heads, best of "
                                         f"{reps} ({secs:.1f} s of fp64 work)"}
    return out


# ------------------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores; each step one bounded sample."""
    if rank != 0:
        return None
    import oracle as oracle_pkg
    cfg = PREFILL_CFG
    orc = oracle_pkg.get()
    # each step about 1.5 s of oracle work, so K + W steps end within a few minutes
    b_rows, t_tok = sized_sample(cfg, 1.5)
    a, u, s0, _ = oracle_sample(cfg, b_rows, t_tok)
    nthreads = oracle_pkg.default_threads()
    for _ in range(args.warmup):
        orc.prefill(*a, u, s0, nthreads=nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.prefill(*a, u, s0, nthreads=nthreads)
    dt = time.perf_counter() - t0
    value = b_rows * t_tok * args.steps / dt
    sample = f"{b_rows} batch row x {t_tok} tokens x {cfg.H} heads per step, fp64"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "wkv6_prefill_1p5b_layer", "B": cfg.B, "T": cfg.T, "H": cfg.H,
                   "D": cfg.D, "io": "bf16 inputs, fp64 arithmetic"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--algo", choices=["auto", "recurrent", "chunked"], default="auto")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-other", action="store_true",
                    help="skip the long-context and decay-extreme prefill lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clock-warm", action="store_true",
                    help="skip the ~1 s untimed warm-up loop (for profiler runs)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the prefill batch size (smaller profiler captures)")
    ap.add_argument("--only", choices=["backward", "backward_c2", "gold", "extreme_ln"],
                    default=None,
                    help="print only that line (wkv6_backward, or GOLD compression + "
                         "decompression, on the 1.5B-layer shape; or the decay-extreme prefill "
                         "with LayerNorm; --batch and --seq-len override B and T), for "
                         "profiler runs")
    ap.add_argument("--seq-len", type=int, default=None, help="T of --only")
    ap.add_argument("--seqpar", action="store_true",
                    help="print only the long-context shape as one sequence split across the "
                         "ranks (NCCL exchange; a process group is set up even at one rank)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        # host-only arm: rank 0 runs the oracle and prints; other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    world, rank, local = dist_setup()
    try:
        if args.seqpar:
            import torch.distributed as dist
            from linear_attention_rnn_finch_b200 import binding
            binding.load()
            dev = torch.device("cuda", local)
            if not dist.is_initialized():   # one rank: a one-member NCCL group
                import datetime
                import socket
                with socket.socket() as sk:
                    sk.bind(("127.0.0.1", 0))
                    port = sk.getsockname()[1]
                dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                        world_size=1, timeout=datetime.timedelta(seconds=120),
                                        device_id=dev)
                world = 1
            hbm, _ = peaks()
            out = seqpar_line(dev, world, rank, args.steps, hbm)
        elif args.only is not None:
            from linear_attention_rnn_finch_b200 import binding
            binding.load()
            base = W.CONFIGS[4] if args.only == "extreme_ln" else PREFILL_CFG
            cfg = base.with_(**{k: v for k, v in (("B", args.batch), ("T", args.seq_len))
                                if v is not None})
            dev = torch.device("cuda", local)
            hbm, _ = peaks()
            out = (gold_line(dev, world, steps=args.steps, B=cfg.B, T=cfg.T)
                   if args.only == "gold" else
                   other_prefill(cfg, dev, world, hbm, args.algo, steps=args.steps)
                   if args.only == "extreme_ln" else
                   backward_line(cfg, dev, world, steps=args.steps,
                                 c2=args.only == "backward_c2"))
        else:
            out = run_ours(args, world, rank, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
