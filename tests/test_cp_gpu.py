"""Context parallelism across devices (kda_cp_local_map, all-gather, kda_cp_finish)
emulated on one GPU: the ranks' steps run one after another in one process (no
kernel waits on another), with the "all-gather" a stack of the ranks' maps.  The
concatenated outputs, every rank's starting state and the last rank's final state
must match the fp64 oracle on the whole sequence (rel-L2 <= 1e-2, max-abs <= 5e-2)."""
import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF16 = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _check(got, ref, what):
    x = got.detach().double().cpu().numpy()
    r = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    m = float(np.abs(x - ref).max())
    assert r <= 1e-2 and m <= 5e-2, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def _emulate(inp, world):
    B, T, H, dk = inp["q"].shape
    Tl = T // world
    sl = lambda x, r: x[:, r * Tl:(r + 1) * Tl].contiguous()  # noqa: E731
    wss, maps = [], []
    for r in range(world):
        ws = torch.empty(kda.cp_workspace_size(B, Tl, H, dk, dk, BF16), dtype=torch.uint8,
                         device=DEV)
        maps.append(kda.kda_cp_local_map(sl(inp["q"], r), sl(inp["k"], r), sl(inp["v"], r),
                                         sl(inp["g"], r), sl(inp["beta"], r), workspace=ws))
        wss.append(ws)
    gathered = torch.stack(maps)
    outs, s_ins, hT = [], [], None
    for r in range(world):
        o = torch.empty(B, Tl, H, dk, dtype=BF16, device=DEV)
        hT = torch.empty(B, H, dk, dk, device=DEV)
        _, _, s_in = kda.kda_cp_finish(gathered, r, inp["h0"], B=B, T_local=Tl, H=H, dk=dk,
                                       dv=dk, dtype=BF16, o=o, hT=hT, workspace=wss[r])
        outs.append(o)
        s_ins.append(s_in)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    return torch.cat(outs, dim=1), s_ins, hT


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("case", ["workload", "no_decay"])
def test_emulated_ranks_match_the_whole_sequence(world, case):
    # 768 tokens: divisible by every world size tested (stretches of whole chunks)
    inp = W.make_prefill_inputs(2, 64 * 12, 2, 128, 128, BF16, True, seed=70 + world,
                                device=DEV)
    if case == "no_decay":      # nothing forgets: every rank's start carries everything
        inp["g"][..., 0::2] = 0.0
    o, s_ins, hT = _emulate(inp, world)
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["h0"])
    _check(o, o_ref, f"world {world} {case} o")
    _check(hT, hT_ref, f"world {world} {case} hT")
    Tl = inp["q"].shape[1] // world
    for r in range(1, world):   # rank r starts from the state after r stretches
        pre = lambda x: x[:, :r * Tl].contiguous()  # noqa: E731
        _, s_ref = oracle.kda_fwd(pre(inp["q"]), pre(inp["k"]), pre(inp["v"]), pre(inp["g"]),
                                  pre(inp["beta"]), inp["h0"])
        _check(s_ins[r], s_ref, f"world {world} rank {r} starting state")


def test_rank_zero_needs_no_maps_and_ragged_local_stretch():
    """Rank 0 folds nothing (maps may be absent); a local stretch that is not a
    multiple of the 64-token chunk ends in a partial chunk."""
    inp = W.make_prefill_inputs(1, 100, 3, 128, 128, BF16, True, seed=80, device=DEV)
    ws = torch.empty(kda.cp_workspace_size(1, 100, 3, 128, 128, BF16), dtype=torch.uint8,
                     device=DEV)
    m = kda.kda_cp_local_map(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], workspace=ws)
    o = torch.empty(1, 100, 3, 128, dtype=BF16, device=DEV)
    hT = torch.empty(1, 3, 128, 128, device=DEV)
    kda.kda_cp_finish(m[None], 0, inp["h0"], B=1, T_local=100, H=3, dk=128, dv=128, dtype=BF16,
                      o=o, hT=hT, workspace=ws)
    torch.cuda.synchronize()
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    _check(o, o_ref, "rank 0 o")
    _check(hT, hT_ref, "rank 0 hT")
    # the map itself: R is the stretch's final state from zero
    _, r_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None)
    _check(m[..., :128], r_ref, "R of the local map")
