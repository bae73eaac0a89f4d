"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Tolerances (whole-tensor relative L2, and elementwise max-abs for bf16), for
outputs o and final states separately:
  * fp32 q/k/v:  rel-L2 <= 1e-4
  * bf16 q/k/v:  rel-L2 <= 1e-2 and max-abs <= 5e-2 (fp32 state)
Inputs come from the seeded generators in ``kimi_delta_attention_28_b200.workloads``;
the oracle sees exactly the values the kernels see (bf16 and fp32 widen to fp64
exactly).
"""
import math

import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def rel_l2(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return float(np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-300))


def assert_close(got, ref, dtype, what=""):
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else np.asarray(got)
    r = rel_l2(got, ref)
    m = float(np.abs(got - ref).max()) if got.size else 0.0
    if dtype == torch.float32:
        assert r <= 1e-4, f"{what}: rel-L2 {r:.3e} > 1e-4"
    else:
        assert r <= 1e-2 and m <= 5e-2, f"{what}: rel-L2 {r:.3e} (<=1e-2), max-abs {m:.3e} (<=5e-2)"
    return r, m


def run_and_check(inp, dtype, what):
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        inp["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["h0"], inp["cu_seqlens"])
    assert_close(o, o_ref, dtype, what + " o")
    assert_close(hT, hT_ref, dtype, what + " hT")
    return o, hT


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def test_tiny_fp32_workload():
    w = W.TINY
    inp = W.make_workload(w, DEV)
    run_and_check(inp, w.dtype, w.name)


def test_prefill_workload_full_size():
    w = W.PREFILL
    inp = W.make_workload(w, DEV)
    run_and_check(inp, w.dtype, w.name)


@pytest.mark.parametrize("T", [1, 15, 63, 64, 65, 127, 200, 1000])
@pytest.mark.parametrize("h0", [False, True])
def test_ragged_lengths_tensor_core_path(T, h0):
    inp = W.make_prefill_inputs(2, T, 3, 128, 128, torch.bfloat16, h0, seed=T * 7 + h0, device=DEV)
    run_and_check(inp, torch.bfloat16, f"bf16 T={T}")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_head_sizes_and_dtypes(d, dtype):
    inp = W.make_prefill_inputs(2, 77, 2, d, d, dtype, True, seed=d, device=DEV)
    run_and_check(inp, dtype, f"{dtype} d={d}")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_varlen_small_with_empty_sequences(dtype, d):
    lengths = [5, 0, 64, 1, 130, 0, 77]
    inp = W.make_prefill_inputs(1, 0, 3, d, d, dtype, True, seed=3, device=DEV, lengths=lengths)
    run_and_check(inp, dtype, "varlen small")


@pytest.mark.parametrize("T", [64, 130])
def test_many_chains_several_waves(T):
    """512 (sequence, head) chains: more than two waves of 32-column state slices,
    so the state pass runs on 64-column slices (eight state warps per CTA)."""
    inp = W.make_prefill_inputs(64, T, 8, 128, 128, torch.bfloat16, True, seed=T + 17, device=DEV)
    run_and_check(inp, torch.bfloat16, f"512 chains T={T}")


def test_varlen_workload_sampled_heads():
    """Packed varlen workload (16 sequences, H=32) on the GPU; the oracle checks
    every sequence on a sample of heads (heads are independent chains)."""
    w = W.VARLEN
    inp = W.make_workload(w, DEV)
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        inp["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    for h in (0, 19):
        sl = lambda x: x[:, :, h:h + 1].contiguous()  # noqa: E731
        o_ref, hT_ref = oracle.kda_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                       inp["beta"][:, :, h:h + 1].contiguous(),
                                       inp["h0"][:, h:h + 1].contiguous(), inp["cu_seqlens"])
        assert_close(o[:, :, h:h + 1], o_ref, w.dtype, f"varlen head {h} o")
        assert_close(hT[:, h:h + 1], hT_ref, w.dtype, f"varlen head {h} hT")


def test_long_context_workload_windows():
    """1M-token workload (B=1, H=16).  Every transition has operator norm
    <= max_c exp(g_tc), so a run restarted from zero L tokens before a position
    differs from the full run by at most exp(sum of per-token max g) times the
    state norm; with L = 4096 that factor is computed from the data and must be
    negligible.  Sampled output blocks and the final state are checked against
    oracle runs on such windows."""
    w = W.LONG
    inp = W.make_workload(w, DEV)
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    T, L, blk = w.T, 4096, 64
    gmax = inp["g"][0].amax(dim=-1)   # [T, H]: per-token largest log-decay
    rng = np.random.default_rng(0)
    starts = sorted(rng.integers(L, T - blk, size=3).tolist()) + [T - blk]
    # crude state-norm bound: ||S_t|| <= sum_u beta_u |k_u| |v_u| <= t * max|v| * sqrt(d_v)
    snorm = T * float(inp["v"].abs().max()) * math.sqrt(w.dv)
    for s in starts:
        a = s - L
        factor = math.exp(float(gmax[a:s].sum(dim=0).max()))
        assert factor * snorm < 1e-8, "window too short for the truncation bound"
        sl = lambda x: x[:, a:s + blk].contiguous()  # noqa: E731
        o_ref, hT_ref = oracle.kda_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                       sl(inp["beta"]), None)
        assert_close(o[:, s:s + blk], o_ref[:, L:], w.dtype, f"long o[{s}:{s + blk}]")
        if s + blk == T:
            assert_close(hT, hT_ref, w.dtype, "long hT")


def test_decode_workload():
    """256 sequences x 96 heads: the full state after one step against the
    oracle, then 1000 chained steps checked on 64 sampled (sequence, head) chains."""
    w = W.DECODE
    steps = w.decode_steps
    inp = W.make_workload(w, DEV, steps=steps)
    S = inp["S"].clone()
    S0 = inp["S"]
    o1 = kda.kda_decode_step(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0], S)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.kda_decode_step(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0],
                                          inp["beta"][0], S0)
    assert_close(o1, o_ref, w.dtype, "decode step 1 o")
    assert_close(S, S_ref, w.dtype, "decode step 1 S")
    rng = np.random.default_rng(1)
    pairs = rng.choice(w.B * w.H, size=64, replace=False)
    n_idx = torch.tensor(pairs // w.H, device=DEV)
    h_idx = torch.tensor(pairs % w.H, device=DEV)
    outs = [o1[n_idx, h_idx]]
    for t in range(1, steps):
        o_t = kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                  inp["beta"][t], S)
        outs.append(o_t[n_idx, h_idx])
    torch.cuda.synchronize()
    pick = lambda x: x[:, n_idx, h_idx].unsqueeze(2).transpose(0, 1).contiguous()  # [64, steps, 1, d]  # noqa: E731
    o_ref, S_ref = oracle.kda_fwd(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["g"]),
                                  inp["beta"][:, n_idx, h_idx].transpose(0, 1).unsqueeze(2).contiguous(),
                                  S0[n_idx, h_idx].unsqueeze(1).contiguous())
    o_all = torch.stack(outs).transpose(0, 1).unsqueeze(2)
    assert_close(o_all, o_ref, w.dtype, "decode 1000 steps o")
    assert_close(S[n_idx, h_idx].unsqueeze(1), S_ref, w.dtype, "decode 1000 steps S")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_small_and_chained_equals_prefill(d, dtype):
    N, H, steps = 3, 2, 9
    inp = W.make_decode_inputs(N, H, d, d, steps, dtype, seed=d + 1, device=DEV)
    S = inp["S"].clone()
    outs = [kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                inp["beta"][t], S) for t in range(steps)]
    torch.cuda.synchronize()
    tr = lambda x: x.transpose(0, 1).contiguous()  # [steps, N, ...] -> [N, steps, ...]  # noqa: E731
    o_ref, S_ref = oracle.kda_fwd(tr(inp["q"]), tr(inp["k"]), tr(inp["v"]), tr(inp["g"]),
                                  tr(inp["beta"]), inp["S"])
    assert_close(tr(torch.stack(outs)), o_ref, dtype, "decode chain o")
    assert_close(S, S_ref, dtype, "decode chain S")


def test_in_place_state_update():
    inp = W.make_prefill_inputs(2, 300, 2, 128, 128, torch.bfloat16, True, seed=5, device=DEV)
    h0 = inp["h0"].clone()
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], h0)
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        hT=inp["h0"])
    torch.cuda.synchronize()
    assert hT.data_ptr() == inp["h0"].data_ptr()
    assert_close(hT, hT_ref, torch.bfloat16, "in-place hT")
    assert_close(o, o_ref, torch.bfloat16, "in-place o")


def test_no_final_state_and_zero_length():
    inp = W.make_prefill_inputs(1, 100, 2, 128, 128, torch.bfloat16, True, seed=6, device=DEV)
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        output_final_state=False)
    torch.cuda.synchronize()
    assert hT is None
    o_ref, _ = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    assert_close(o, o_ref, torch.bfloat16, "no-final-state o")
    e = W.make_prefill_inputs(2, 0, 2, 128, 128, torch.bfloat16, True, seed=7, device=DEV)
    o, hT = kda.kda_fwd(e["q"], e["k"], e["v"], e["g"], e["beta"], e["h0"])
    torch.cuda.synchronize()
    assert torch.equal(hT, e["h0"])


def test_phases_compose_to_fwd_bitwise():
    # (at these sizes kda_fwd runs the two launches, not the overlapped one)
    assert not kda.plan_overlap(2, 500, 4, 128, 128, 0, torch.bfloat16)
    inp = W.make_prefill_inputs(2, 500, 4, 128, 128, torch.bfloat16, True, seed=8, device=DEV)
    o1, h1 = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    ws = torch.empty(kda.workspace_size(2, 500, 4, 128, 128, 0, torch.bfloat16),
                     dtype=torch.uint8, device=DEV)
    kda.kda_fwd_intra(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], workspace=ws)
    o2 = torch.empty_like(o1)
    h2 = torch.empty_like(h1)
    kda.kda_fwd_inter(inp["h0"], None, o2, h2, B=2, T=500, H=4, dk=128, dv=128,
                      dtype=torch.bfloat16, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_deterministic():
    inp = W.make_prefill_inputs(2, 333, 3, 128, 128, torch.bfloat16, True, seed=9, device=DEV)
    a = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    b = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("cu", [[0, 10, 5, 20], [1, 10, 20], [0, 10, 19]])
def test_bad_offsets_are_reported_and_write_nothing(cu):
    T = 20
    inp = W.make_prefill_inputs(1, T, 2, 128, 128, torch.bfloat16, True, seed=10, device=DEV)
    cu_t = torch.tensor(cu, dtype=torch.int32, device=DEV)
    N = len(cu) - 1
    o = torch.full((1, T, 2, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    hT = torch.full((N, 2, 128, 128), 7.0, dtype=torch.float32, device=DEV)
    h0 = torch.zeros(N, 2, 128, 128, device=DEV)
    kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], h0, cu_t, o=o, hT=hT)
    assert kda.device_error() == 7      # KDA_ERR_BAD_SEQLENS, read and cleared
    assert kda.device_error() == 0
    assert bool((o == 7.0).all()) and bool((hT == 7.0).all())


def test_extreme_decay_at_the_bound():
    """g within 1e-3 of the stated lower bound -5 everywhere: the sub-tile
    reference points must keep every factor finite."""
    inp = W.make_prefill_inputs(1, 256, 2, 128, 128, torch.bfloat16, True, seed=11, device=DEV)
    inp["g"] = -5.0 + 1e-3 * torch.rand_like(inp["g"])
    o, hT = run_and_check(inp, torch.bfloat16, "g at bound")
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()


@pytest.mark.parametrize("case", ["no_decay", "no_write", "full_write", "mixed_decay"])
def test_special_inputs_tensor_core_path(case):
    """Corner values of the gates over 4,096 tokens (64 chunks, several record
    rings' worth): g = 0 (nothing forgets, the state carries everything), beta = 0
    (pure decay of h0, no writes), beta = 1 (full delta-rule overwrite), and
    channels that never decay next to channels at the decay bound."""
    inp = W.make_prefill_inputs(1, 4096, 2, 128, 128, torch.bfloat16, True, seed=12, device=DEV)
    if case == "no_decay":
        inp["g"].zero_()
    elif case == "no_write":
        inp["beta"].zero_()
    elif case == "full_write":
        inp["beta"].fill_(1.0)
    else:
        inp["g"][..., 0::2] = 0.0
        inp["g"][..., 1::2] = -5.0
    o, hT = run_and_check(inp, torch.bfloat16, case)
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
