"""The prefill and decode entry points inside CUDA graphs.

They allocate nothing and never synchronise, so a stream capture of them replays
as a graph: the graph is replayed on new input values (copied into the captured
buffers) and each replay is checked against the oracle."""
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


# two launches; time-split policy; the overlapped single launch (ready flags cleared by a
# captured memset, the cooperative kernel captured as a graph node)
@pytest.mark.parametrize("shape", [(2, 1000, 4), (1, 20000, 1), (2, 8192, 8)])
def test_prefill_graph_replays_on_new_inputs(shape):
    B, T, H = shape
    if shape == (2, 8192, 8) and not kda.plan_overlap(B, T, H, 128, 128, 0, BF16):
        pytest.skip("kda_fwd does not overlap at these sizes on this GPU")
    bufs = W.make_prefill_inputs(B, T, H, 128, 128, BF16, True, seed=90, device=DEV)
    ws = torch.empty(kda.workspace_size(B, T, H, 128, 128, 0, BF16), dtype=torch.uint8,
                     device=DEV)
    o = torch.empty_like(bufs["v"])
    hT = torch.empty_like(bufs["h0"])
    args = (bufs["q"], bufs["k"], bufs["v"], bufs["g"], bufs["beta"], bufs["h0"])
    kda.kda_fwd(*args, o=o, hT=hT, workspace=ws)          # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        kda.kda_fwd(*args, o=o, hT=hT, workspace=ws)
    for seed in (91, 92):
        new = W.make_prefill_inputs(B, T, H, 128, 128, BF16, True, seed=seed, device=DEV)
        for name in ("q", "k", "v", "g", "beta", "h0"):
            bufs[name].copy_(new[name])
        graph.replay()
        torch.cuda.synchronize()
        assert kda.device_error() == 0
        o_ref, hT_ref = oracle.kda_fwd(new["q"], new["k"], new["v"], new["g"], new["beta"],
                                       new["h0"], None)
        assert_close(o, o_ref, BF16, f"graph replay seed {seed} o")
        assert_close(hT, hT_ref, BF16, f"graph replay seed {seed} hT")


def test_decode_steps_in_one_graph():
    steps, N, H = 8, 4, 3
    inp = W.make_decode_inputs(N, H, 128, 128, steps, BF16, seed=93, device=DEV)
    S0 = inp["S"].clone()
    S = inp["S"].clone()
    outs = [torch.empty(N, H, 128, dtype=BF16, device=DEV) for _ in range(steps)]
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        for t in range(steps):
            kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                inp["beta"][t], S, o=outs[t])
    graph.replay()
    torch.cuda.synchronize()
    S_ref = S0
    for t in range(steps):
        o_ref, S_ref = oracle.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t],
                                              inp["g"][t], inp["beta"][t], S_ref)
        assert_close(outs[t], o_ref, BF16, f"graph decode step {t} o")
    assert_close(S, S_ref, BF16, "graph decode final state")
