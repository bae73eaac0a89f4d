"""Context parallelism across ranks on CPU: two and three gloo processes, as torchrun
would start them, each holding one stretch of the same sequences.  Each rank
summarises its stretch as the affine map [R | P] of the recurrence -- computed here
by the fp64 oracle (R: the stretch run from a zero state; P: run from the identity
with zero values, the linear part) -- the library's gather_segment_maps exchanges the
maps in rank order, and each rank folds the maps of the ranks before it onto the
initial state.  Every rank's starting state and the last rank's final state must
equal the oracle's run over the whole sequence.  (The GPU kernels of the same
steps are checked on one device by tests/test_cp_gpu.py.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from kimi_delta_attention_28_b200 import _lib


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed=5, B=2, T=36, H=2, d=4):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, d))
    g = -0.3 / (1.0 + np.exp(-rng.standard_normal((B, T, H, d))))   # slow decay: big carries
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    h0 = 0.5 * rng.standard_normal((B, H, d, d))
    return q, k, v, g, beta, h0


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, g, beta, h0 = _inputs()
        B, T, H, d = q.shape
        Tl = T // world
        sl = lambda x: x[:, rank * Tl:(rank + 1) * Tl]  # noqa: E731
        # this rank's map [R | P] per (sequence, head)
        _, R = oracle.kda_fwd(sl(q), sl(k), sl(v), sl(g), sl(beta), None)
        eye = np.broadcast_to(np.eye(d), (B, H, d, d)).copy()
        _, P = oracle.kda_fwd(sl(q), sl(k), np.zeros_like(sl(v)), sl(g), sl(beta), eye)
        local = torch.from_numpy(np.concatenate([R, P], axis=-1))
        maps = _lib.gather_segment_maps(local).numpy()          # [world, B, H, d, 2d]
        S = h0.copy()
        for s in range(rank):                                   # prefix combine
            S = maps[s, ..., d:] @ S + maps[s, ..., :d]
        S_end = maps[rank, ..., d:] @ S + maps[rank, ..., :d]
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, S, S_end, maps.shape))
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_combine_to_the_whole_sequence(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, g, beta, h0 = _inputs()
    B, T, H, d = q.shape
    Tl = T // world
    for rank, S, S_end, shape in res:
        assert shape == (world, B, H, d, 2 * d)
        pre = lambda x: x[:, :rank * Tl]  # noqa: E731
        _, S_ref = oracle.kda_fwd(pre(q), pre(k), pre(v), pre(g), pre(beta), h0)
        assert np.allclose(S, S_ref, rtol=1e-10, atol=1e-10), rank
        upto = lambda x: x[:, :(rank + 1) * Tl]  # noqa: E731
        _, E_ref = oracle.kda_fwd(upto(q), upto(k), upto(v), upto(g), upto(beta), h0)
        assert np.allclose(S_end, E_ref, rtol=1e-10, atol=1e-10), rank
