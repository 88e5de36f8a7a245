"""The N > 1 host logic of the benchmark, as two `gloo` ranks on the CPU: every rank gets
its own batch of the same shape, the step time reported is the maximum over ranks, and the
reference arm runs on rank 0 alone (the others leave without work)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(workloads.WORKLOADS["v3_decode_b32_ctx4096"], rank)
        bench.barrier()
        m = bench.max_over_ranks(1.5 + rank)          # rank r "took" 1.5 + r ms
        args = type("A", (), {"steps": 1, "warmup": 0, "reference_seconds": 0.0})()
        ref_rc = bench.run_reference(args, w) if rank != 0 else None
        q.put((rank, w.name, w.seed, w.B, w.ctx, m, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    (r0, n0, s0, b0, c0, m0, _), (r1, n1, s1, b1, c1, m1, ref1) = got
    assert (b0, c0) == (b1, c1) == (32, 4096)     # same shape on every rank (weak scaling)
    assert s0 != s1                                # but its own inputs
    assert m0 == m1 == 2.5                         # the max over ranks, seen by all
    assert ref1 == 0                               # non-zero ranks leave the reference arm at once


def test_single_rank_helpers_without_a_process_group():
    assert bench.max_over_ranks(3.0) == 3.0
    w = workloads.WORKLOADS["v3_decode_b32_ctx4096"]
    assert bench.rank_workload(w, 0) is w
