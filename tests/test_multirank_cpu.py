"""The multi-rank path of bench.py on CPU: two gloo ranks (no GPU).

Every rank runs its own seeded copy of the workload (independent problems, weak
scaling); the only cross-rank traffic is the barrier and the max-over-ranks of
the step time. This checks both, the per-rank inputs, the whole-job value, and
that the reference arm does no work on ranks other than 0.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench
    import sa_workloads as W
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slowest
        slowest = bench.rank_max(ms, world, "cpu")
        w = bench.workload_params("gzip_8k", rank, "small")
        q = W.qkv(w, "q", 0, head=0)[:64]
        args = type("A", (), dict(workload="gzip_8k", steps=1, warmup=0, gpus=world))()
        ref = bench.run_reference(args) if rank == 1 else None  # must return at once
        # every workload's copy on this rank, and a level-2 gist of the gist-of-gist decode
        idx = {n: bench.workload_params(n, rank, "full")["index"]
               for n in ("gist_coarse_20k", "gist_hier_decode_128k", "gzip_flags_128m", "gist_decode_128k")}
        g2 = W.decode_gists2(bench.workload_params("gist_hier_decode_128k", rank, "small"), 0, "k")[0, :4]
        out[rank] = dict(slowest=slowest, index=w["index"], q=q, ref=ref, idx=idx, g2=g2,
                         value=bench.weak_scaling_value(1e12, world, slowest, 1e12))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        r0, r1 = out[0], out[1]
    assert r0["slowest"] == r1["slowest"] == 15.0
    assert r0["index"] != r1["index"]                 # independent problems
    assert not np.array_equal(r0["q"], r1["q"])       # different seeded inputs
    assert r1["ref"] is None                          # reference arm: rank 0 only
    assert all(r1["idx"][n] == r0["idx"][n] + 1000 for n in r0["idx"])
    assert not np.array_equal(r0["g2"], r1["g2"])
    assert r0["value"] == pytest.approx(2 / 15e-3)    # all ranks' work / slowest time
