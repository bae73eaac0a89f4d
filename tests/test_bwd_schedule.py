"""The segmented backward's bookkeeping, exhaustively on the CPU.

Three kernels meet at segment boundaries through checkpoint slots, and the slot
arithmetic lives in device code; this test restates it and checks, for every length
and segment size, that each segment reads the state the forward stored at its first
token and the state gradient the reversed chain stored at its last.
  - state pass with checkpoints every `every` chunks (kda_prefill_tc.cuh): after `done`
    chunks of sequence n, if done % every == 0 and done * 64 <= T, slot
    n * floor(T / (64 every)) + done / every - 1;
  - the reversed chain is the same pass over the chunks in reverse order, so its
    `done` counts chunks from the end: the slot holds dL/dS at boundary cps - done;
  - the slice kernel (kda_bwd.cuh), segment s of sc chunks: start state slot
    n nfw + s - 1 (s > 0), end gradient slot n nfw + cps / sc - s - 2 (s < nseg - 1),
    nfw = floor(T / (64 sc)).
"""
import pytest

C = 64


def forward_slots(N, T, every):
    cps = -(-T // C)
    per = T // (C * every)
    slots = {}
    for n in range(N):
        for done in range(1, cps + 1):
            if done % every == 0 and done * C <= T:
                slots[n * per + done // every - 1] = (n, done)      # state after `done` chunks
    return slots


def reverse_slots(N, T, every):
    cps = -(-T // C)
    per = T // (C * every)
    slots = {}
    for n in range(N):
        for done in range(1, cps + 1):
            if done % every == 0 and done * C <= T:
                slots[n * per + done // every - 1] = (n, cps - done)   # gradient at that boundary
    return slots


@pytest.mark.parametrize("T", list(range(65, 1300, 37)) + [128, 256, 4096, 4160])
def test_segments_read_their_boundaries(T):
    N = 3
    cps = -(-T // C)
    for sc in range(1, cps):
        if cps % sc:
            continue
        nseg, nfw = cps // sc, T // (C * sc)
        fwd, rev = forward_slots(N, T, sc), reverse_slots(N, T, sc)
        cap = N * nfw
        assert all(0 <= k < cap for k in fwd) and all(0 <= k < cap for k in rev)
        for n in range(N):
            for s in range(nseg):
                if s > 0:
                    assert fwd[n * nfw + s - 1] == (n, s * sc), (T, sc, n, s)
                if s < nseg - 1:
                    assert rev[n * nfw + cps // sc - s - 2] == (n, (s + 1) * sc), (T, sc, n, s)
