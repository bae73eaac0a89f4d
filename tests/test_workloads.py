"""The synthetic input recipe (CPU): what the seeded generators draw, and the shapes of
the named workloads.  The tests and the bench both take their inputs from here."""
import math

import torch

from kimi_delta_attention_28_b200 import workloads as W


def test_prefill_input_distributions():
    inp = W.make_prefill_inputs(2, 300, 3, 64, 32, torch.bfloat16, True, seed=5)
    q, k, v, g, beta, h0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "h0"))
    assert q.shape == k.shape == g.shape == (2, 300, 3, 64) and v.shape == (2, 300, 3, 32)
    assert beta.shape == (2, 300, 3) and h0.shape == (2, 3, 64, 32)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    assert g.dtype == beta.dtype == h0.dtype == torch.float32
    assert inp["cu_seqlens"] is None
    # q, k L2-normalised per (token, head), q also scaled by 1/sqrt(d_k) (bf16-rounded)
    assert torch.allclose(k.float().norm(dim=-1), torch.ones(2, 300, 3), atol=1e-2)
    assert torch.allclose(q.float().norm(dim=-1), torch.full((2, 300, 3), 1 / math.sqrt(64)),
                          atol=2e-3)
    # g = -5 sigmoid(z), z ~ N(-3, 1): inside (-5, 0), mean near -5 sigmoid(-3) ~ -0.25
    assert (g < 0).all() and (g > -5).all()
    assert -0.45 < g.mean().item() < -0.15
    assert ((beta > 0) & (beta < 1)).all() and abs(beta.mean().item() - 0.5) < 0.05
    assert abs(v.float().std().item() - 1.0) < 0.05
    assert abs(h0.std().item() - 0.1) < 0.005          # "N(0, 0.1)": standard deviation 0.1


def test_generators_are_deterministic_by_seed():
    a = W.make_prefill_inputs(1, 100, 2, 32, 32, torch.float32, True, seed=11)
    b = W.make_prefill_inputs(1, 100, 2, 32, 32, torch.float32, True, seed=11)
    c = W.make_prefill_inputs(1, 100, 2, 32, 32, torch.float32, True, seed=12)
    for n in ("q", "k", "v", "g", "beta", "h0"):
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])
    d1 = W.make_decode_inputs(3, 2, 32, 32, 4, torch.bfloat16, seed=3)
    d2 = W.make_decode_inputs(3, 2, 32, 32, 4, torch.bfloat16, seed=3)
    assert all(torch.equal(d1[n], d2[n]) for n in d1)
    assert d1["q"].shape == (4, 3, 2, 32) and d1["S"].shape == (3, 2, 32, 32)


def test_varlen_lengths_and_offsets():
    lens = W.varlen_lengths(16, 1024, 32768, seed=1003)
    assert lens == W.varlen_lengths(16, 1024, 32768, seed=1003)
    assert all(1024 <= n <= 32768 for n in lens) and len(set(lens)) > 8
    cu = W.cu_from_lengths(lens)
    assert cu.dtype == torch.int32 and cu[0] == 0 and cu[-1] == sum(lens)
    assert bool((cu[1:] >= cu[:-1]).all())
    inp = W.make_prefill_inputs(1, 0, 2, 32, 32, torch.bfloat16, True, seed=4,
                                lengths=[5, 0, 70])
    assert inp["q"].shape == (1, 75, 2, 32) and inp["h0"].shape == (3, 2, 32, 32)
    assert inp["cu_seqlens"].tolist() == [0, 5, 5, 75]


def test_named_workloads():
    assert (W.TINY.B, W.TINY.H, W.TINY.T, W.TINY.dk, W.TINY.dtype) == (1, 2, 64, 32, torch.float32)
    assert not W.TINY.h0
    assert (W.PREFILL.B, W.PREFILL.H, W.PREFILL.T, W.PREFILL.dk) == (2, 8, 4096, 128)
    assert W.PREFILL.h0 and W.PREFILL.dtype == torch.bfloat16
    assert (W.LONG.B, W.LONG.H, W.LONG.T, W.LONG.dk) == (1, 16, 1 << 20, 128) and not W.LONG.h0
    assert (W.VARLEN.varlen_seqs, W.VARLEN.H, W.VARLEN.varlen_range) == (16, 32, (1024, 32768))
    assert (W.DECODE.B, W.DECODE.H, W.DECODE.dk, W.DECODE.decode_steps) == (256, 96, 128, 1000)
    assert len({w.seed for w in W.ALL}) == len(W.ALL)
