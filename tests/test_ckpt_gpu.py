"""State checkpoints at token boundaries (kda_fwd_checkpointed) against the oracle.

For prefix caching a prefill also stores each sequence's state after every
`ckpt_every` tokens.  The reference for checkpoint c of a sequence is the fp64
oracle run over that sequence's first (c + 1) * ckpt_every tokens, obtained here by
running the oracle over consecutive pieces of `ckpt_every` tokens, each from the
previous piece's final state (the split-run property the oracle's own pins check).
o and hT must be bitwise those of kda_fwd.
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W
from tests.test_parity_gpu import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BF16 = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _sequences(inp):
    """(q, k, v, g, beta, h0) per sequence, each [L, H, d] (h0 [1, H, dk, dv] or None)."""
    q, cu = inp["q"], inp["cu_seqlens"]
    if cu is None:
        bounds = [(n, 0, q.shape[1]) for n in range(q.shape[0])]
    else:
        c = cu.tolist()
        bounds = [(0, c[n], c[n + 1]) for n in range(len(c) - 1)]
    out = []
    for i, (b, t0, t1) in enumerate(bounds):
        sl = lambda x: x[b, t0:t1]  # noqa: E731
        h0 = None if inp["h0"] is None else inp["h0"][i:i + 1]
        out.append((sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]), h0))
    return out


def _checkpoint_oracle(inp, every):
    H, dk, dv = inp["q"].shape[2], inp["q"].shape[3], inp["v"].shape[3]
    refs = []
    for q, k, v, g, beta, h0 in _sequences(inp):
        S = h0
        for c in range(q.shape[0] // every):
            p = slice(c * every, (c + 1) * every)
            _, S, _ = oracle.kda_fwd_packed(q[p], k[p], v[p], g[p], beta[p], S)
            refs.append(S[0])
    return np.stack(refs) if refs else np.zeros((0, H, dk, dv))


def _run(inp, every, **kw):
    o, hT, ck = kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                         inp["h0"], inp["cu_seqlens"], ckpt_every=every, **kw)
    o1, hT1 = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                          inp["cu_seqlens"])
    torch.cuda.synchronize()
    return o, hT, ck, o1, hT1


@pytest.mark.parametrize("every", [64, 128, 320])
def test_fixed_length_checkpoints(every):
    """B=2, T=1,000 (a ragged last chunk), nonzero h0."""
    inp = W.make_prefill_inputs(2, 1000, 2, 128, 128, BF16, True, seed=70 + every, device=DEV)
    o, hT, ck, o1, hT1 = _run(inp, every)
    assert kda.device_error() == 0
    assert torch.equal(o, o1) and torch.equal(hT, hT1)
    assert ck.shape == (2 * (1000 // every), 2, 128, 128)
    assert_close(ck, _checkpoint_oracle(inp, every), BF16, f"checkpoints every {every}")


def test_packed_checkpoints_with_short_and_empty_sequences():
    lengths = [300, 0, 700, 64, 129]          # 4, 0, 10, 1, 2 checkpoints at 64
    inp = W.make_prefill_inputs(1, 0, 2, 128, 128, BF16, True, seed=75, device=DEV,
                                lengths=lengths)
    o, hT, ck, o1, hT1 = _run(inp, 64)
    assert kda.device_error() == 0
    assert torch.equal(o, o1) and torch.equal(hT, hT1)
    assert ck.shape[0] == sum(n // 64 for n in lengths) == 17
    assert_close(ck, _checkpoint_oracle(inp, 64), BF16, "packed checkpoints")


def test_checkpoints_through_the_time_split():
    """One chain of 64 chunks: kda_fwd splits the state pass in time by itself, and the
    checkpoints come from the output pass of every segment."""
    inp = W.make_prefill_inputs(1, 4096, 1, 128, 128, BF16, True, seed=77, device=DEV)
    inp["g"][..., ::4] = 0.0                  # undecayed channels carry state across segments
    assert kda.plan_segments(1, 4096, 1, 128, 128, 0, BF16) > 1
    o, hT, ck, o1, hT1 = _run(inp, 256)
    assert kda.device_error() == 0
    assert torch.equal(o, o1) and torch.equal(hT, hT1)
    assert_close(ck, _checkpoint_oracle(inp, 256), BF16, "checkpoints, split state pass")
    # the last checkpoint is the final state
    assert torch.equal(ck[-1], hT[0])


def test_packed_capacity_overflow_is_reported():
    lengths = [300, 700]                      # 4 + 10 checkpoints at 64
    inp = W.make_prefill_inputs(1, 0, 2, 128, 128, BF16, True, seed=78, device=DEV,
                                lengths=lengths)
    ck = torch.full((5, 2, 128, 128), 3.0, device=DEV)
    kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                             inp["cu_seqlens"], ckpt_every=64, ckpts=ck)
    assert kda.device_error() == 9            # KDA_ERR_CHECKPOINT_CAPACITY
    assert kda.device_error() == 0
    assert_close(ck, _checkpoint_oracle(inp, 64)[:5], BF16, "slots within the capacity")


def test_host_checks():
    inp = W.make_prefill_inputs(1, 512, 2, 128, 128, BF16, True, seed=79, device=DEV)
    args = (inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    with pytest.raises(ValueError):
        kda.kda_fwd_checkpointed(*args, ckpt_every=100)
    with pytest.raises(kda.KDAError) as e:    # 512 // 128 = 4 slots needed
        kda.kda_fwd_checkpointed(*args, ckpt_every=128,
                                 ckpts=torch.empty(3, 2, 128, 128, device=DEV))
    assert e.value.code == 1
