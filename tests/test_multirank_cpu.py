"""bench.py's N > 1 host logic on CPU: two gloo ranks on 127.0.0.1.

The path shards by batch with no data-path collective: each rank runs its own batch of the
workload (its own seed), the job's time is the slowest rank's and its token count the sum
over ranks.  Checked here: the process-group set-up, max / sum over ranks, that the ranks'
inputs differ, that rank-sharded oracle results equal one run over the stacked batch, and
that the reference arm does no work on ranks other than 0.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import argparse
    import bench
    import oracle
    from linear_attention_rnn_finch_b200 import workloads as W
    import torch.distributed as dist

    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    mx = bench.max_over_ranks(10.0 + rank, world)
    sm = bench.sum_over_ranks(1.0 + rank, world)
    bench.barrier(world)
    # each rank's shard: a small batch of the prefill workload with the rank's seed
    cfg = W.CONFIGS[1].with_(B=1, T=40, H=2)
    inp = W.make_prefill_shard(cfg, "cpu", rank)
    f = lambda t: t.to(torch.float64).numpy()
    y, s = oracle.get().prefill(*[f(inp[n]) for n in ("r", "k", "v", "omega")], f(inp["u"]),
                                f(inp["state0"]), nthreads=1)
    ref = bench.run_reference(argparse.Namespace(steps=1, warmup=3), world, rank)
    np.savez(os.path.join(outdir, f"rank{rank}.npz"), mx=mx, sm=sm, y=y, s=s,
             r=f(inp["r"]), k=f(inp["k"]), v=f(inp["v"]), omega=f(inp["omega"]),
             u=f(inp["u"]), s0=f(inp["state0"]), ref_none=(ref is None) if rank else True)
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path, oracle):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    d = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    for x in d:
        assert float(x["mx"]) == 11.0 and float(x["sm"]) == 3.0
        assert bool(x["ref_none"])
    assert not np.array_equal(d[0]["r"], d[1]["r"])   # ranks draw different batches
    # the ranks' shards are independent: one run over the stacked batch gives the same
    cat = {n: np.concatenate([x[n] for x in d]) for n in ("r", "k", "v", "omega", "s0")}
    assert np.array_equal(d[0]["u"], d[1]["u"])        # shared parameter, same per rank
    y, s = oracle.prefill(cat["r"], cat["k"], cat["v"], cat["omega"], d[0]["u"], cat["s0"])
    assert np.array_equal(y, np.concatenate([x["y"] for x in d]))
    assert np.array_equal(s, np.concatenate([x["s"] for x in d]))
