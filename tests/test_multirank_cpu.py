"""The multi-rank (N > 1) host path on CPU: two `gloo` ranks on 127.0.0.1.

bench.py runs one process per GPU, each an independent replica batch (weak
scaling, no data-path collective), and reports the slowest rank's time. These
tests cover the host logic of that path without a GPU: the max-over-ranks
reduction, per-rank inputs, and that (batch, head) slices sharded across ranks
and gathered give exactly the single-process oracle result (the independence
the sharding relies on).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, results):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from oracle import dark_oracle as O
        from random_feature_linear_b200 import synth

        out = {}
        # slowest rank's time on every rank
        out["max"] = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
        # replica inputs: same shapes, different draws per rank
        w = synth.WORKLOADS[2].with_sizes(B=2, H=4, L=96, lengths=(96, 70))
        mine = synth.make_inputs(w, salt=rank)
        out["q_shape"] = mine["q"].shape
        out["q_sum"] = float(np.abs(mine["q"]).sum())
        # heads sharded round-robin over ranks, gathered: the oracle per shard
        base = synth.make_inputs(w)
        heads = [h for h in range(w.H) if h % WORLD == rank]
        part = O.attention(base["q"][:, heads], base["k"][:, heads], base["v"][:, heads],
                           base["omega"], base["geom"][heads], key_mask=base["mask"],
                           causal=True)[0]
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, (heads, part))
        full = np.zeros_like(base["q"], dtype=np.float64)
        for hs, o in gathered:
            full[:, hs] = o
        ref = O.attention(base["q"], base["k"], base["v"], base["omega"], base["geom"],
                          key_mask=base["mask"], causal=True)[0]
        out["shard_err"] = float(np.abs(full - ref).max())
        results[rank] = out
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.start_processes(_rank_main, args=(port, results), nprocs=WORLD, join=True,
                       start_method="spawn")
    r0, r1 = results[0], results[1]
    assert r0["max"] == r1["max"] == 2.5
    assert r0["q_shape"] == r1["q_shape"]
    assert r0["q_sum"] != r1["q_sum"]
    assert r0["shard_err"] == 0.0 and r1["shard_err"] == 0.0


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
