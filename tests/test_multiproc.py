"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
each, rendezvous on 127.0.0.1) check that the reported time is the slowest
rank's, that the whole-job value counts every rank's work (weak scaling: each
rank owns the same number of units of a global problem), that the ranks' (batch,
KV-head) units are disjoint and together cover the global batch, and that
ranks draw different seeded batches of the same shape. No GPU and no kernel is
involved; the kernels need no exchange between ranks (each (batch, KV head)
unit is independent)."""
import os
import socket

import numpy as np
import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    import bench
    from exact_io_aware_45_b200 import inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        got = bench.max_over_ranks(ms)
        x = inputs.random_case(1, 2, 1, 64, 16, seed=rank)
        units = bench.rank_units(world, rank, B=4, Hkv=8)
        gathered = [None] * world
        dist.all_gather_object(gathered, units)
        out.put((rank, got, float(np.sum(x["q"])), x["q"].shape, gathered))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, sh0, u0), (r1, t1, s1, sh1, u1) = res
    assert t0 == t1 == 15.0                         # max over ranks on every rank
    assert sh0 == sh1 and s0 != s1                  # same per-rank shape, different batches
    assert u0 == u1                                 # both ranks see the same partition
    a, b = set(u0[0]), set(u0[1])
    assert len(a) == len(b) == 4 * 8 and not (a & b)
    assert a | b == {(bb, hk) for bb in range(2 * 4) for hk in range(8)}


def test_job_value_is_weak_scaling():
    import bench
    # 2 ranks, 3 steps of 1e12 FLOP each per rank, slowest rank 2 s -> 3 TFLOP/s
    assert bench.job_tflops(1e12, 3, 2, 2000.0) == pytest.approx(3.0)
    assert bench.max_over_ranks(7.5) == 7.5         # no process group: unchanged
