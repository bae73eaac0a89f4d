"""The time-split state pass (kda_fwd_segmented, and kda_fwd's own split policy)
against the fp64 oracle.

Every chunk's map on the state is affine, S -> P S + R, so a chain cut into
segments can be summarised segment by segment ([R | P] from zero / identity),
combined in prefix order and rerun from the true segment starting states.
These tests check that the result is the unsplit recurrence: against the oracle
with the bf16 tolerances of the other parity tests, and against the unsplit
CUDA pass (the two differ only by rounding in the carried state).
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W
from tests.test_parity_gpu import assert_close, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BF16 = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _oracle(inp):
    return oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                          inp["cu_seqlens"])


def _split(inp, nseg, **kw):
    o, hT = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  inp["h0"], inp["cu_seqlens"], num_segments=nseg, **kw)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    return o, hT


@pytest.mark.parametrize("nseg", [1, 2, 3, 7, 16])
@pytest.mark.parametrize("T", [1000, 4096])
def test_segments_match_oracle_and_unsplit(nseg, T):
    inp = W.make_prefill_inputs(2, T, 2, 128, 128, BF16, True, seed=50 + nseg, device=DEV)
    o, hT = _split(inp, nseg)
    o_ref, hT_ref = _oracle(inp)
    assert_close(o, o_ref, BF16, f"T={T} nseg={nseg} o")
    assert_close(hT, hT_ref, BF16, f"T={T} nseg={nseg} hT")
    o1, hT1 = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    torch.cuda.synchronize()
    plain_policy = (kda.workspace_size(2, T, 2, 128, 128, 0, BF16)
                    == kda.segmented_workspace_size(2, T, 2, 128, 128, 0, BF16, 1))
    if nseg == 1 and plain_policy:   # kda_fwd does not split either: bit for bit
        assert torch.equal(o, o1) and torch.equal(hT, hT1)
    else:   # as accurate as the plain pass
        for got, plain, ref in ((o, o1, o_ref), (hT, hT1, hT_ref)):
            r_split = rel_l2(got.double().cpu(), ref)
            assert r_split <= 1.5 * rel_l2(plain.double().cpu(), ref) + 5e-4


def test_more_segments_than_chunks_and_empty_sequences():
    """Packed batch whose short sequences have fewer chunks than segments (empty
    trailing segments: P = I, R = 0) and empty sequences (hT = h0)."""
    lengths = [700, 0, 5, 64, 1, 1500, 0, 129]
    inp = W.make_prefill_inputs(1, 0, 3, 128, 128, BF16, True, seed=61, device=DEV,
                                lengths=lengths)
    o, hT = _split(inp, 8)
    o_ref, hT_ref = _oracle(inp)
    assert_close(o, o_ref, BF16, "varlen nseg=8 o")
    assert_close(hT, hT_ref, BF16, "varlen nseg=8 hT")


def test_in_place_state_with_segments():
    inp = W.make_prefill_inputs(1, 2000, 2, 128, 128, BF16, True, seed=62, device=DEV)
    o_ref, hT_ref = _oracle(inp)
    S = inp["h0"].clone()
    inp2 = dict(inp, h0=S)
    o, hT = _split(inp2, 5, hT=S)
    assert hT.data_ptr() == S.data_ptr()
    assert_close(o, o_ref, BF16, "in-place o")
    assert_close(S, hT_ref, BF16, "in-place hT")


def test_zero_decay_channels_carry_state_through_segments():
    """g = 0 on half the key channels: nothing decays there, so the state carried
    across segment boundaries (the P part of each map) is far from zero and the
    combine has real work to do."""
    inp = W.make_prefill_inputs(1, 3000, 2, 128, 128, BF16, True, seed=63, device=DEV)
    inp["g"][..., ::2] = 0.0
    o, hT = _split(inp, 6)
    o_ref, hT_ref = _oracle(inp)
    assert_close(o, o_ref, BF16, "g=0 channels o")
    assert_close(hT, hT_ref, BF16, "g=0 channels hT")


def test_auto_policy_splits_few_long_chains():
    """B=1, H=1, T=16,384: one chain of 256 chunks would run on one SM's worth of
    CTAs; kda_fwd splits it by itself.  The workspace it asks for includes the
    split's buffers, and the result matches the oracle and the explicit split."""
    B, T, H = 1, 16384, 1
    assert kda.plan_segments(B, T, H, 128, 128, 0, BF16) > 1
    assert kda.plan_segments(2, 4096, 8, 128, 128, 0, BF16) == 1   # 16 chains fill the GPU
    plain = kda.segmented_workspace_size(B, T, H, 128, 128, 0, BF16, 1)
    auto = kda.workspace_size(B, T, H, 128, 128, 0, BF16)
    assert auto > plain   # room for the split
    inp = W.make_prefill_inputs(B, T, H, 128, 128, BF16, True, seed=64, device=DEV)
    # Undecayed channels keep state alive across segment boundaries, so the split
    # path's rounding differs from the plain pass (with the workload's decays the
    # carried state underflows within a segment and both paths agree bit for bit).
    inp["g"][..., ::4] = 0.0
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    o_ref, hT_ref = _oracle(inp)
    assert_close(o, o_ref, BF16, "auto split o")
    assert_close(hT, hT_ref, BF16, "auto split hT")
    o1, hT1 = _split(inp, 1)
    assert not torch.equal(o, o1)   # the split path really ran (different rounding)
    # and it is as accurate as the plain pass
    for got, plain, ref, what in ((o, o1, o_ref, "o"), (hT, hT1, hT_ref, "hT")):
        r_split = rel_l2(got.double().cpu(), ref)
        r_plain = rel_l2(plain.double().cpu(), ref)
        assert r_split <= 1.5 * r_plain + 5e-4, (what, r_split, r_plain)


def test_bad_segment_counts():
    inp = W.make_prefill_inputs(1, 100, 1, 128, 128, BF16, False, seed=65, device=DEV)
    for bad in (0, -1, 4097):
        with pytest.raises(kda.KDAError):
            _split(inp, bad)
    f32 = W.make_prefill_inputs(1, 100, 1, 64, 64, torch.float32, False, seed=66, device=DEV)
    with pytest.raises(kda.KDAError):
        _split(f32, 2)
    o, hT = _split(f32, 1)   # one segment: any path
    o_ref, hT_ref = _oracle(f32)
    assert_close(o, o_ref, torch.float32, "fp32 nseg=1 o")
