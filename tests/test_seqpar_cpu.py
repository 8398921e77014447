"""Sequence parallelism's host logic on CPU: one long sequence split over two gloo ranks on
127.0.0.1 (linear_attention_rnn_finch_b200/seqpar.py).  The device steps are replaced by
fp64 oracle computations of what they define (the summary: the state a span builds from a
zero state and its total log2 decay; the carry; the prefill of a span from its incoming
state); the exchange is the module's own all-gather.  The two ranks' outputs, joined, must
equal one oracle run over the whole sequence, and both ranks must report its final state.
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, T_SPAN, H, D = 2, 48, 2, 64


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_sequence():
    from linear_attention_rnn_finch_b200 import workloads as W
    cfg = W.CONFIGS[1].with_(seed=9600, B=B, T=2 * T_SPAN, H=H)
    return W.make_prefill_inputs(cfg, "cpu")


class OracleOps:
    """The device steps as the oracle computes them (host-only test double)."""

    def __init__(self, orc):
        self.o = orc

    @staticmethod
    def f(t):
        return t.to(torch.float64).numpy()

    def summary(self, k, v, omega):
        z = np.zeros(k.shape)
        _, s = self.o.prefill(z, self.f(k), self.f(v), self.f(omega), np.zeros((H, D)), None,
                              nthreads=1)
        g = (-np.exp(self.f(omega))).sum(axis=1) / np.log(2.0)   # [B, H, D] log2 decay
        return torch.from_numpy(s), torch.from_numpy(g)

    def exchange(self, s_loc, g, group):
        from linear_attention_rnn_finch_b200.seqpar import GpuOps
        return GpuOps().exchange(s_loc, g, group)

    def carry(self, all_s, all_g, state0):
        P = all_s.shape[0]
        s = np.zeros((B, H, D, D)) if state0 is None else self.f(state0)
        out = [s]
        for p in range(P):
            s = np.exp2(all_g[p].numpy())[..., None] * s + all_s[p].numpy()
            out.append(s)
        return torch.from_numpy(np.stack(out))

    def prefill(self, r, k, v, omega, u, state_in, ln):
        y, s = self.o.prefill(self.f(r), self.f(k), self.f(v), self.f(omega), self.f(u),
                              self.f(state_in), nthreads=1)
        return torch.from_numpy(y), torch.from_numpy(s)


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from linear_attention_rnn_finch_b200 import seqpar

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    inp = _full_sequence()
    span = slice(rank * T_SPAN, (rank + 1) * T_SPAN)
    a = [inp[n][:, span].contiguous() for n in ("r", "k", "v", "omega")]
    y, s = seqpar.prefill_sequence_parallel(*a, inp["u"], inp["state0"],
                                            ops=OracleOps(oracle.get()))
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), y=y.numpy(), s=s.numpy())
    dist.destroy_process_group()


def test_two_gloo_ranks_split_one_sequence(tmp_path, oracle):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    d = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    inp = _full_sequence()
    f = lambda t: t.to(torch.float64).numpy()
    y, s = oracle.prefill(*[f(inp[n]) for n in ("r", "k", "v", "omega", "u", "state0")])
    y_joined = np.concatenate([x["y"] for x in d], axis=1)
    scale = np.abs(y).max()
    assert np.abs(y_joined - y).max() <= 1e-12 * scale
    for x in d:   # every rank holds the final state of the whole sequence
        assert np.abs(x["s"] - s).max() <= 1e-12 * np.abs(s).max()
