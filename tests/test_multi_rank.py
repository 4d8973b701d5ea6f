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


def _shard_worker(rank, world, port, q):
    """One problem split by KV-head group: each rank plans its own groups
    (host logic only) and the ranks check together that their items cover
    every (query row, group) pair once and that their output rows are
    disjoint."""
    import numpy as np
    import sparse_long_context_nsa_b200 as nsa
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seqs, n1, n2, d1, d2, l, d, lp, count = (3000, 700, 0, 1500), 32, 4, 64, 64, 32, 16, 64, 8
        cuq = np.cumsum(seqs).astype(np.int32)
        cuc = nsa.nsa_compress_out_len(cuq, l, d)
        cus = np.cumsum([-(-s // lp) for s in seqs]).astype(np.int32)
        b, c = nsa.nsa_shard_groups(n2, world, rank)
        items = nsa.nsa_compress_attention_shard_plan(n1, n2, d1, d2, l, d, lp, count, cuq, cuc, cus, b, c)
        t1 = int(cuq[-1])
        cover = torch.zeros(t1, n2, dtype=torch.int64)
        heads = torch.zeros(t1, n1, dtype=torch.int64)     # attention_out / stats rows this rank writes
        G = n1 // n2
        for row0, ntok, g in items:
            cover[row0:row0 + ntok, g] += 1
            heads[row0:row0 + ntok, g * G:(g + 1) * G] += 1
        dist.all_reduce(cover)
        dist.all_reduce(heads)
        q.put((rank, b, c, bool((cover == 1).all()), bool((heads == 1).all())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_one_problem_by_head_group():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(o[1], o[2]) for o in out] == [(0, 2), (2, 2)]
    assert all(o[3] for o in out), "every (query row, KV group) pair computed by exactly one rank"
    assert all(o[4] for o in out), "every output row written by exactly one rank"
