"""The multi-process plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them.  Each rank works on its own batch (weak scaling: the seed is
offset by the rank), and the job time is the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # slowest rank wins
        t = bench.max_over_ranks(1.5 + rank, world, "cpu")
        # each rank draws its own batch of the bench workload
        w, inp = bench.workload_inputs("prefill", "cpu", seed_offset=rank)
        digest = float(inp["q"][0, :8].float().sum()) + float(inp["g"][0, :8].sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, t, w.seed, digest))
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = out.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.5, 2.5]          # max over ranks on every rank
    assert res[0][2] != res[1][2]                      # per-rank seeds
    assert res[0][3] != res[1][3]                      # so different inputs


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
