"""The data-parallel (weak-scaling) path with two ranks on the CPU over gloo: each rank runs its
own independently seeded workload, with no exchange on the data path; the only collectives are
the timing barrier, the max of the ranks' times and the sum of their token counts."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from paged_block_quantized_b200 import workloads as W
        from _oracle_run import oracle_step
        w = W.make("tiny", seed=100 + rank)             # this rank's own shard of sequences
        o = oracle_step(w)                              # the step on this shard alone
        fake_time = 1.0 + rank                          # rank 1 is the slower one
        bench.dist_barrier(world)
        t_max = bench.dist_max(fake_time, world)
        tok = bench.dist_sum(float(w.total_tokens), world)
        out[rank] = (t_max, tok, float(w.total_tokens), o["out"].sum(), all(e == 0 for e in o["errors"]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 2.0                  # every rank sees the slowest rank's time
    assert r0[1] == r1[1] == r0[2] + r1[2]        # tokens of both shards, whole job
    assert r0[3] != r1[3]                         # the shards are different problems
    assert r0[4] and r1[4]
