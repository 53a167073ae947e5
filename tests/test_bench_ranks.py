"""The multi-GPU path of the benchmark on the CPU: two gloo ranks (one
process per rank, rendezvous on 127.0.0.1).  Replicas only: the job's time is
the slowest rank's, the reference arm runs on rank 0 alone, and the workload
description counts every rank's canvases."""

import argparse
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    slowest = bench.max_over_ranks(1.5 + rank, world)
    args = argparse.Namespace(workload="full", steps=1, warmup=0)
    wl = bench.WORKLOADS["full"]
    cfg = bench.workload_config(args, wl, world)
    # the reference arm runs on rank 0 only: the other ranks leave at once
    ref_rc = bench.reference_arm(args, wl, rank, world) if rank != 0 else 0
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, slowest, cfg["global_batch"], cfg["parallelism"], ref_rc))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [2.5, 2.5]          # max over ranks, seen by both
    assert all(g[2] == 2 and g[3] == "replicas x2" for g in got)
    assert got[1][4] == 0                             # rank 1: reference arm returns without work


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
