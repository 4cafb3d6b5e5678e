"""The multi-GPU path's host logic, as two gloo ranks on the CPU.

Token batches are independent, so bench.py runs one replica per rank (weak
scaling, no data-path collective): each rank draws its own seeded batch, the
timed region is bracketed by a barrier, the reported time is the maximum over
ranks, and only rank 0 prints.  These tests run those pieces with world size 2
over gloo at 127.0.0.1."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from w4a4_post_quantized_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank reports its own elapsed time; the job's is the maximum
        elapsed = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(world, elapsed)
        # each rank's batch comes from its own seed (seed = 1000 * rank + ...)
        x = synth.activations(64, 1024, seed=1000 * rank + 10)
        # the reference arm runs on rank 0 only; the others return at once
        class A:
            cpu_rows = 16; steps = 1; warmup = 0
        out = None
        if rank != 0:
            out = bench.run_reference(A, bench.WORKLOADS["c1_single_linear"], world, rank)
        bench.barrier(world)
        q.put((rank, mx, int(x.view(np.uint16)[:8].astype(np.int64).sum()), out))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_on_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 15.0 for r in res)          # max over ranks, seen by every rank
    assert res[0][2] != res[1][2]                  # different batches per rank
    assert res[1][3] is None                       # non-zero ranks run no reference work
