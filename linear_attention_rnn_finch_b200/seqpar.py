"""One long sequence split across the ranks of a process group (sequence parallelism).

The recurrence carries a state from one span of tokens to the next, and carrying it
reproduces the single pass (GoldFinch review page, section 3.4 "Training and Inference
Procedures": pre-fill through the recurrence, in parallel chunks).  So a sequence too long
for one GPU's time budget is cut into one span per rank:

    rank p holds tokens [p*T, (p+1)*T) of every (b,h) sequence (T a multiple of 64);
    1. summary: the state its tokens build from a zero state, S_p, and each channel's total
       log2 decay over them, g_p (wkv6_segment_summary, on the tensor cores);
    2. exchange: one all-gather of (S_p, g_p), B*H*(D*D + D) fp32 per rank;
    3. carry: the state entering every span, s_in[p+1] = diag(2^g_p) s_in[p] + S_p
       (wkv6_segment_carry; each rank computes the whole short chain itself);
    4. prefill of its own tokens from s_in[p] (wkv6_prefill, any of its paths).

The only collective is step 2.  The initial state, u and the LayerNorm parameters must be
the same on every rank.  The device work is the library's; this module only orders the
calls and the exchange.  ``ops`` replaces the four steps (the host-only tests substitute
their own), and must implement summary, exchange, carry and prefill as ``GpuOps`` does.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


class GpuOps:
    """The four steps on the GPU through libgoldwkv, the exchange through torch.distributed
    (NCCL between GPUs)."""

    def summary(self, k, v, omega):
        return binding.segment_summary(k, v, omega)

    def exchange(self, s_loc, g, group):
        """All ranks' (s_loc, g), stacked rank-major: one all-gather of both, packed."""
        world = dist.get_world_size(group)
        flat = torch.cat([s_loc.reshape(-1), g.reshape(-1)])
        parts = [torch.empty_like(flat) for _ in range(world)]
        dist.all_gather(parts, flat, group=group)
        n = s_loc.numel()
        all_s = torch.stack([q[:n].view_as(s_loc) for q in parts])
        all_g = torch.stack([q[n:].view_as(g) for q in parts])
        return all_s, all_g

    def carry(self, all_s, all_g, state0):
        return binding.segment_carry(all_s, all_g, state0)

    def prefill(self, r, k, v, omega, u, state_in, ln):
        return binding.wkv6_prefill(r, k, v, omega, u, state_in, ln=ln)


def prefill_sequence_parallel(r, k, v, omega, u, state0=None, *, ln=None, group=None,
                              ops=None):
    """This rank's span of one long sequence.  r, k, v, omega [B, T, H, D] bf16 are this
    rank's tokens (rank p: tokens p*T .. (p+1)*T - 1 of the whole sequence); u [H, D] and
    state0 [B, H, D, D] (or None: zero) are the same on every rank.  Returns (y, state):
    y [B, T, H, D] of this rank's tokens and the state after the whole sequence (the same
    on every rank).  Every rank must call it, with the same shapes."""
    ops = GpuOps() if ops is None else ops
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    s_loc, g = ops.summary(k, v, omega)
    all_s, all_g = ops.exchange(s_loc, g, group)
    assert all_s.shape[0] == world
    s_in = ops.carry(all_s, all_g, state0)
    y, _ = ops.prefill(r, k, v, omega, u, s_in[rank].contiguous(), ln)
    return y, s_in[world]
