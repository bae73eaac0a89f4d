"""Speculative decoding through the C ABI: kda_decode_verify runs K drafted tokens
per (sequence, head) from the state without changing it; kda_decode_commit advances
the state over the accepted prefix only.  Checked against the fp64 oracle (the
recurrence over the drafted tokens / over the accepted prefix) at the parity
tolerances (bf16: rel-L2 <= 1e-2 and max-abs <= 5e-2; fp32: rel-L2 <= 1e-4), and
against the single-token decode step they stand in for."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _check(got, ref, dtype, what):
    x = got.detach().double().cpu().numpy()
    r = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    m = float(np.abs(x - ref).max()) if x.size else 0.0
    if dtype == torch.float32:
        assert r <= 1e-4, f"{what}: rel-L2 {r:.3e}"
    else:
        assert r <= 1e-2 and m <= 5e-2, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def _draft(N, K, H, d, dtype, seed):
    """Drafted tokens in [N, K, H, d] layout (the prefill recipe) and states."""
    inp = W.make_prefill_inputs(N, K, H, d, d, dtype, True, seed=seed, device=DEV)
    return inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"]


@pytest.mark.parametrize("K", [1, 4, 8, 16])
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16),
                                     (32, torch.float32), (128, torch.float32)])
def test_verify_then_commit_every_accepted_length(K, d, dtype):
    N, H = K + 1, 3                      # sequence n accepts n tokens: 0 .. K
    q, k, v, g, beta, S0 = _draft(N, K, H, d, dtype, seed=100 * K + d)
    S = S0.clone()
    o = torch.full((N, K, H, d), float("nan"), dtype=dtype, device=DEV)
    kda.kda_decode_verify(q, k, v, g, beta, S, o)
    torch.cuda.synchronize()
    assert torch.equal(S, S0), "verify must not change the state"
    _check(o, oracle.kda_decode_verify(q, k, v, g, beta, S0), dtype, f"verify K={K} o")
    acc = torch.arange(N, dtype=torch.int32, device=DEV)
    kda.kda_decode_commit(k, v, g, beta, acc, S)
    assert kda.device_error() == 0
    S_ref = oracle.kda_decode_commit(k, v, g, beta, acc, S0)
    assert torch.equal(S[0], S0[0]), "accepting nothing leaves the state as it was"
    _check(S, S_ref, dtype, f"commit K={K} S")


def test_verify_and_full_commit_equal_chained_decode_steps():
    N, K, H, d = 4, 6, 2, 128
    q, k, v, g, beta, S0 = _draft(N, K, H, d, torch.bfloat16, seed=7)
    o = kda.kda_decode_verify(q, k, v, g, beta, S0)
    S_steps = S0.clone()
    steps = [kda.kda_decode_step(q[:, t].contiguous(), k[:, t].contiguous(),
                                 v[:, t].contiguous(), g[:, t].contiguous(),
                                 beta[:, t].contiguous(), S_steps) for t in range(K)]
    S_commit = S0.clone()
    kda.kda_decode_commit(k, v, g, beta, torch.full((N,), K, dtype=torch.int32, device=DEV),
                          S_commit)
    torch.cuda.synchronize()
    o_steps = torch.stack(steps, dim=1)
    # same fp32 arithmetic token by token: agreement far inside the tolerance
    assert float((o.float() - o_steps.float()).abs().max()) <= 2 ** -7
    assert float((S_commit - S_steps).abs().max()) <= 1e-5


def test_bad_accepted_count_is_reported_and_leaves_that_state():
    N, K, H, d = 3, 4, 2, 128
    q, k, v, g, beta, S0 = _draft(N, K, H, d, torch.bfloat16, seed=8)
    S = S0.clone()
    acc = torch.tensor([2, 5, -1], dtype=torch.int32, device=DEV)     # 5 > K, -1 < 0
    kda.kda_decode_commit(k, v, g, beta, acc, S)
    assert kda.device_error() == 11                                   # KDA_ERR_BAD_ACCEPTED
    assert kda.device_error() == 0
    assert torch.equal(S[1:], S0[1:])
    S_ref = oracle.kda_decode_commit(k[:1], v[:1], g[:1], beta[:1], np.array([2]), S0[:1])
    _check(S[:1], S_ref, torch.bfloat16, "valid sequence committed")


def test_decode_workload_shapes_draft_of_four():
    """256 sequences x 96 heads (the decode workload), K = 4 drafted tokens, accepted
    counts 0..4 drawn per sequence: every output and state against the oracle."""
    w = W.DECODE
    K = 4
    inp = W.make_prefill_inputs(w.B, K, w.H, w.dk, w.dv, w.dtype, True, seed=w.seed + 1,
                                device=DEV)
    S0 = inp["h0"]
    S = S0.clone()
    o = kda.kda_decode_verify(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S)
    gen = torch.Generator(device="cpu").manual_seed(5)
    acc = torch.randint(0, K + 1, (w.B,), generator=gen, dtype=torch.int32).to(DEV)
    kda.kda_decode_commit(inp["k"], inp["v"], inp["g"], inp["beta"], acc, S)
    assert kda.device_error() == 0
    _check(o, oracle.kda_decode_verify(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0),
           w.dtype, "workload verify o")
    _check(S, oracle.kda_decode_commit(inp["k"], inp["v"], inp["g"], inp["beta"], acc, S0),
           w.dtype, "workload commit S")
