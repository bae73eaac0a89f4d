"""The backward pass (kda_bwd, kda_bwd_segmented) through the C ABI against the fp64
oracle gradient.

The loss is L = sum(do * o) + sum(dhT * hT) for seeded upstream gradients do (in
the dtype of q) and dhT (fp32).  The per-chain pass computes in fp32 from the exact
input values, so there the gradients stored in fp32 (dg, dbeta, dh0) must match the
fp64 oracle to rel-L2 <= 1e-4 whatever the input dtype; gradients stored in the input
dtype (dq, dk, dv) carry its rounding: rel-L2 <= 1e-4 for fp32 and, for bf16, rel-L2
<= 1e-2 with max-abs <= 5e-2 of the tensor's largest magnitude (at least 1).  The
segmented pass (bf16, d = 128) starts its segments from states of the bf16 tensor-core
forward and ends them at gradients carried over the bf16 chunk records, so every one of
its gradients is held to that bf16 bound, the prefill's own.
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _check(got, ref, stored_dtype, what):
    x = got.detach().double().cpu().numpy()
    assert np.isfinite(x).all(), f"{what}: non-finite values"
    r = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    m = float(np.abs(x - ref).max()) if x.size else 0.0
    scale = max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
    if stored_dtype == torch.float32:
        assert r <= 1e-4, f"{what}: rel-L2 {r:.3e}"
    else:
        assert r <= 1e-2 and m <= 5e-2 * scale, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"
    return r


def _upstream(inp, seed, with_dhT):
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    gen = torch.Generator(device=DEV).manual_seed(seed)
    do = torch.randn(B, T, H, dv, generator=gen, device=DEV).to(inp["q"].dtype)
    dhT = (0.1 * torch.randn(N, H, dk, dv, generator=gen, device=DEV)) if with_dhT else None
    return do, dhT


def _call(inp, do, dhT, num_segments):
    """kda_bwd (num_segments None) or kda_bwd_segmented; returns the gradients and the
    segments per sequence the call used."""
    B, T, H, dk = inp["q"].shape
    cu = inp["cu_seqlens"]
    a = (inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], cu, do, dhT)
    plan = kda.bwd_plan_segments(B, T, H, dk, inp["v"].shape[-1],
                                 0 if cu is None else cu.numel() - 1, inp["q"].dtype)
    if num_segments is None:
        got = kda.kda_bwd(*a)
    else:
        got = kda.kda_bwd_segmented(*a, num_segments=num_segments)
        plan = num_segments or plan
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    return got, plan


def _compare(got, ref, dt, segmented):
    for name, a, b in zip(NAMES, got, ref):
        if a is None:
            continue
        stored = dt if name in ("dq", "dk", "dv") or segmented else torch.float32
        _check(a, b.reshape(a.shape), stored, name)


def _run(inp, seed, with_dhT=True, num_segments=None):
    do, dhT = _upstream(inp, seed, with_dhT)
    got, nseg = _call(inp, do, dhT, num_segments)
    ref = oracle.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do,
                         dhT, inp["cu_seqlens"])
    _compare(got, ref, inp["q"].dtype, nseg >= 2)
    return got


@pytest.mark.parametrize("T", [1, 9, 63, 64, 65, 200])
def test_bf16_d128_ragged_lengths(T):
    inp = W.make_prefill_inputs(2, T, 3, 128, 128, torch.bfloat16, True, seed=T + 40,
                                device=DEV)
    _run(inp, seed=T)


@pytest.mark.parametrize("d,dtype", [(32, torch.float32), (64, torch.float32),
                                     (64, torch.bfloat16), (128, torch.float32)])
def test_head_sizes_and_dtypes(d, dtype):
    inp = W.make_prefill_inputs(2, 77, 2, d, d, dtype, True, seed=d + 7, device=DEV)
    _run(inp, seed=d)


def test_packed_with_empty_sequences_and_no_initial_state():
    inp = W.make_prefill_inputs(1, 0, 2, 128, 128, torch.bfloat16, True, seed=50, device=DEV,
                                lengths=[5, 0, 64, 1, 130, 0, 17])
    _run(inp, seed=51)
    inp["h0"] = None
    got = _run(inp, seed=52, with_dhT=False)
    assert got[5] is None


def test_empty_sequence_passes_the_final_state_gradient_through():
    inp = W.make_prefill_inputs(1, 0, 1, 64, 64, torch.float32, True, seed=53, device=DEV,
                                lengths=[0, 3])
    B, T, H = 1, 3, 1
    do = torch.zeros(B, T, H, 64, device=DEV)
    dhT = torch.randn(2, H, 64, 64, device=DEV)
    got = kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                      inp["cu_seqlens"], do, dhT)
    torch.cuda.synchronize()
    assert torch.equal(got[5][0], dhT[0])


def test_prefill_workload_full_size():
    """The B=2, H=8, T=4,096 workload: every gradient of every token and head, from
    kda_bwd (64 segments of one chunk per sequence) and from the per-chain pass."""
    inp = W.make_workload(W.PREFILL, DEV)
    do, dhT = _upstream(inp, 60, True)
    seg, nseg = _call(inp, do, dhT, None)
    assert nseg == 64
    chain, _ = _call(inp, do, dhT, 1)
    ref = oracle.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do,
                         dhT, None)
    _compare(seg, ref, torch.bfloat16, True)
    _compare(chain, ref, torch.bfloat16, False)


@pytest.mark.parametrize("T", [65, 200])
def test_per_chain_pass_is_exact_for_bf16(T):
    """num_segments = 1: the per-chain fp32 pass, held to 1e-4 on the fp32 gradients."""
    inp = W.make_prefill_inputs(2, T, 3, 128, 128, torch.bfloat16, True, seed=T + 70,
                                device=DEV)
    _run(inp, seed=T + 1, num_segments=1)


@pytest.mark.parametrize("T,nseg,h0,dhT", [(512, 2, True, True), (512, 4, False, True),
                                           (512, 8, True, False), (500, 2, True, True),
                                           (500, 8, False, False), (1000, 16, True, True)])
def test_explicit_segment_counts(T, nseg, h0, dhT):
    """Segments of 1 to 4 chunks (and a ragged last chunk) against the oracle."""
    inp = W.make_prefill_inputs(2, T, 3, 128, 128, torch.bfloat16, h0, seed=T + nseg,
                                device=DEV)
    _run(inp, seed=T + nseg + 1, with_dhT=dhT, num_segments=nseg)


def test_policy_equals_explicit_count():
    inp = W.make_prefill_inputs(1, 200, 2, 128, 128, torch.bfloat16, True, seed=71, device=DEV)
    do, dhT = _upstream(inp, 72, True)
    a, na = _call(inp, do, dhT, None)
    b, _ = _call(inp, do, dhT, na)
    c, _ = _call(inp, do, dhT, 0)
    assert na == 4
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y) and torch.equal(x, z)


def test_explicit_segments_rejected():
    """Counts that do not divide the chunks, other dtypes and head sizes, packed input."""
    def expect_unsupported(inp, n):
        do, dhT = _upstream(inp, 73, True)
        with pytest.raises(kda.KDAError) as e:
            kda.kda_bwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                                  inp["cu_seqlens"], do, dhT, num_segments=n)
        assert e.value.code == 2   # KDA_ERR_UNSUPPORTED_SHAPE
    expect_unsupported(W.make_prefill_inputs(1, 512, 2, 128, 128, torch.bfloat16, True, seed=74,
                                             device=DEV), 3)
    expect_unsupported(W.make_prefill_inputs(1, 512, 2, 128, 128, torch.bfloat16, True, seed=74,
                                             device=DEV), 16)
    expect_unsupported(W.make_prefill_inputs(1, 512, 2, 64, 64, torch.float32, True, seed=75,
                                             device=DEV), 2)
    expect_unsupported(W.make_prefill_inputs(1, 0, 2, 128, 128, torch.bfloat16, True, seed=76,
                                             device=DEV, lengths=[128, 128]), 2)


def test_deterministic():
    inp = W.make_prefill_inputs(1, 150, 2, 128, 128, torch.bfloat16, True, seed=61, device=DEV)
    do = torch.randn(1, 150, 2, 128, device=DEV).to(torch.bfloat16)
    a = kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], None, do)
    b = kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], None, do)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
