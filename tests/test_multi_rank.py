"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank runs an independent batch (seed offset by rank, no collective on
the data path); the timed device time is reduced with a max over ranks; only
rank 0 runs the CPU reference arm.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import bench
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = bench.rank_workload(workloads.TINY.name, rank)
        x = wl.generate()
        # ranks hold different inputs of identical shape
        checksum = float(x["q"].float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (wl.seed, tuple(x["q"].shape), checksum))
        mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank], torch.device("cpu"), world)
        sm = bench.sum_over_ranks([1.0 + rank, 0.5], torch.device("cpu"), world)

        class A:
            workload = workloads.TINY.name
            steps, warmup, ref_rows = 1, 0, 4
        ref_printed = bench.run_reference(A, rank, world) if rank != 0 else "rank0"
        q.put((rank, gathered, mx + sm, ref_printed))
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_batches_and_max_reduction():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    (_, g0, mx0, _), (_, g1, mx1, ref1) = out
    assert g0 == g1
    seeds = [g[0] for g in g0]
    assert seeds[0] != seeds[1]
    assert g0[0][1] == g0[1][1]                 # same shapes
    assert g0[0][2] != g0[1][2]                 # different data
    assert mx0 == mx1 == [2.0, 10.0, 3.0, 1.0]  # max (then sum) over ranks, identical everywhere
    assert ref1 is None                         # reference arm: rank 0 only
