"""Stand-ins for a memory sanitizer on the GPU (compute-sanitizer is closed on this
pool).

NaN canaries: every output buffer (o, final states, checkpoints) and the workspace
are filled with NaN bit patterns before a call; afterwards every output element
must be finite and match the fp64 oracle (bf16 tolerances: rel-L2 <= 1e-2,
max-abs <= 5e-2; fp32: rel-L2 <= 1e-4).  An element the kernels forgot to write,
or a value computed from workspace bytes they never wrote, shows up as NaN.
Shapes are ragged (partial last chunks) and packed inputs include empty sequences.

Debug build: libkda_b200_debug.so carries device-side bounds checks on every
index that addresses global memory; it runs the same small ragged shapes in a
child process (a process loads one copy of the library) and must agree with the
oracle with no check firing, and a workspace whose per-sequence chunk offsets are
corrupted between the two phases must be caught by the checks (status
KDA_ERR_DEBUG_BOUNDS, the affected outputs left untouched) rather than read out
of bounds.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
import oracle
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BF16 = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _check(got, ref, dtype, what):
    x = got.detach().double().cpu().numpy()
    assert np.isfinite(x).all(), f"{what}: {int((~np.isfinite(x)).sum())} elements not written"
    r = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    m = float(np.abs(x - ref).max()) if x.size else 0.0
    if dtype == torch.float32:
        assert r <= 1e-4, f"{what}: rel-L2 {r:.3e}"
    else:
        assert r <= 1e-2 and m <= 5e-2, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def _nan_like(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device=DEV)


def _nan_workspace(nbytes):
    return torch.full((max(nbytes, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes


def _case(kind):
    if kind == "fixed":
        return W.make_prefill_inputs(2, 200, 3, 128, 128, BF16, True, seed=31, device=DEV)
    if kind == "packed":
        return W.make_prefill_inputs(1, 0, 3, 128, 128, BF16, True, seed=32, device=DEV,
                                     lengths=[70, 0, 1, 129, 0, 64])
    if kind == "fp32":
        return W.make_prefill_inputs(2, 45, 2, 64, 64, torch.float32, True, seed=33, device=DEV)
    raise ValueError(kind)


def _outs(inp):
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    N = B if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    return _nan_like((B, T, H, dv), inp["q"].dtype), _nan_like((N, H, dk, dv), torch.float32)


def _ref(inp):
    return oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                          inp["cu_seqlens"])


@pytest.mark.parametrize("kind", ["fixed", "packed", "fp32"])
def test_fwd_writes_every_output(kind):
    inp = _case(kind)
    o, hT = _outs(inp)
    B, T, H, dk = inp["q"].shape
    nseq = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    ws = _nan_workspace(kda.workspace_size(B, T, H, dk, dk, nseq, inp["q"].dtype))
    kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                inp["cu_seqlens"], o=o, hT=hT, workspace=ws)
    assert kda.device_error() == 0
    o_ref, hT_ref = _ref(inp)
    _check(o, o_ref, inp["q"].dtype, f"{kind} o")
    _check(hT, hT_ref, inp["q"].dtype, f"{kind} hT")


def test_overlapped_writes_every_output():
    """The single-launch schedule, with NaN in o, hT and the whole workspace (its ready
    flags and progress counters included: the call clears them itself)."""
    inp = W.make_prefill_inputs(3, 64 * 5 + 9, 2, 128, 128, BF16, True, seed=37, device=DEV)
    o, hT = _outs(inp)
    B, T, H, dk = inp["q"].shape
    ws = _nan_workspace(kda.workspace_size(B, T, H, dk, dk, 0, BF16))
    kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], o=o,
                           hT=hT, workspace=ws)
    assert kda.device_error() == 0
    o_ref, hT_ref = _ref(inp)
    _check(o, o_ref, BF16, "overlapped o")
    _check(hT, hT_ref, BF16, "overlapped hT")


@pytest.mark.parametrize("kind", ["fixed", "packed"])
def test_time_split_writes_every_output(kind):
    inp = W.make_prefill_inputs(1, 64 * 40 + 17, 2, 128, 128, BF16, True, seed=34, device=DEV) \
        if kind == "fixed" else W.make_prefill_inputs(
            1, 0, 2, 128, 128, BF16, True, seed=35, device=DEV, lengths=[64 * 20 + 5, 0, 64 * 9])
    o, hT = _outs(inp)
    B, T, H, dk = inp["q"].shape
    nseq = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    ws = _nan_workspace(kda.segmented_workspace_size(B, T, H, dk, dk, nseq, BF16, 3))
    kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                          inp["cu_seqlens"], num_segments=3, o=o, hT=hT, workspace=ws)
    assert kda.device_error() == 0
    o_ref, hT_ref = _ref(inp)
    _check(o, o_ref, BF16, f"split {kind} o")
    _check(hT, hT_ref, BF16, f"split {kind} hT")


def test_checkpointed_writes_every_checkpoint():
    inp = W.make_prefill_inputs(1, 0, 2, 128, 128, BF16, True, seed=36, device=DEV,
                                lengths=[300, 0, 128, 90])
    o, hT = _outs(inp)
    n_ck = kda.checkpoint_count(0, 128, 1, inp["cu_seqlens"])          # 2 + 1 + 0
    ck = _nan_like((n_ck, 2, 128, 128), torch.float32)
    kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                             inp["cu_seqlens"], ckpt_every=128, ckpts=ck, o=o, hT=hT)
    assert kda.device_error() == 0
    o_ref, hT_ref = _ref(inp)
    _check(o, o_ref, BF16, "ckpt o")
    _check(hT, hT_ref, BF16, "ckpt hT")
    # checkpoint c of sequence n is the state after its first (c + 1) * 128 tokens
    cu = inp["cu_seqlens"].tolist()
    slot = 0
    for n in range(len(cu) - 1):
        for c in range((cu[n + 1] - cu[n]) // 128):
            t1 = cu[n] + (c + 1) * 128
            sl = lambda x: x[:, cu[n]:t1].contiguous()  # noqa: E731
            _, s_ref = oracle.kda_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                      sl(inp["beta"]), inp["h0"][n:n + 1])
            _check(ck[slot:slot + 1], s_ref, BF16, f"checkpoint {slot}")
            slot += 1
    assert slot == n_ck


def test_noalloc_writes_every_output():
    inp = _case("packed")
    o, hT = _outs(inp)
    kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        inp["cu_seqlens"], o, hT)
    assert kda.device_error() == 0
    o_ref, hT_ref = _ref(inp)
    _check(o, o_ref, BF16, "noalloc o")
    _check(hT, hT_ref, BF16, "noalloc hT")


@pytest.mark.parametrize("dtype,d", [(BF16, 128), (torch.float32, 32)])
def test_decode_writes_every_output(dtype, d):
    inp = W.make_decode_inputs(5, 3, d, d, 1, dtype, seed=37, device=DEV)
    S = inp["S"].clone()
    o = _nan_like((5, 3, d), dtype)
    kda.kda_decode_step(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0], S, o)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.kda_decode_step(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0],
                                          inp["beta"][0], inp["S"])
    _check(o, o_ref, dtype, "decode o")
    _check(S, S_ref, dtype, "decode S")


DEBUG_CHILD = textwrap.dedent("""
    import sys, torch, numpy as np
    sys.path.insert(0, %r)
    import kimi_delta_attention_28_b200 as kda, oracle
    from kimi_delta_attention_28_b200 import _lib, workloads as W
    lib = _lib.load_library(_lib.DEBUG_LIB_PATH)
    assert lib.kda_build_flags() == 1, "not the debug build"
    dev = "cuda:0"
    worst = 0.0
    def err(x, y):
        x = x.double().cpu().numpy()
        assert np.isfinite(x).all()
        return max(np.linalg.norm(x - y) / np.linalg.norm(y), np.abs(x - y).max() / 5.0)
    cases = [W.make_prefill_inputs(2, T, 2, 128, 128, torch.bfloat16, True, seed=T, device=dev)
             for T in (1, 63, 65, 200)]
    cases.append(W.make_prefill_inputs(1, 0, 2, 128, 128, torch.bfloat16, True, seed=5,
                                       device=dev, lengths=[70, 0, 1, 129]))
    cases.append(W.make_prefill_inputs(2, 40, 2, 64, 64, torch.float32, True, seed=6, device=dev))
    for inp in cases:
        o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                            inp["cu_seqlens"])
        assert kda.device_error() == 0
        o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                       inp["h0"], inp["cu_seqlens"])
        tol = 1e-2 if inp["q"].dtype == torch.bfloat16 else 1e-4
        worst = max(worst, err(o, o_ref) / tol, err(hT, hT_ref) / tol)
    # the overlapped single launch (its prep workers' and state blocks' checks)
    inp = cases[3]
    o, hT = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    assert kda.device_error() == 0
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    worst = max(worst, err(o, o_ref) / 1e-2, err(hT, hT_ref) / 1e-2)
    inp = W.make_prefill_inputs(1, 64 * 30, 1, 128, 128, torch.bfloat16, True, seed=7, device=dev)
    o, hT = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                                  num_segments=4)
    assert kda.device_error() == 0
    o_ref, hT_ref = oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    worst = max(worst, err(o, o_ref) / 1e-2, err(hT, hT_ref) / 1e-2)
    # corrupt the per-sequence chunk offsets between the phases: the state pass's
    # checks must refuse the two affected sequences and leave their outputs alone
    inp = cases[4]
    B, T, H = inp["q"].shape[:3]
    ws = torch.zeros(kda.workspace_size(B, T, H, 128, 128, 4, torch.bfloat16),
                     dtype=torch.uint8, device=dev)
    kda.kda_fwd_intra(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                      workspace=ws)
    assert kda.device_error() == 0
    # seq_off[0..N] sits 256 bytes into the workspace: seq_off[1] (bytes 260..263) ends
    # sequence 0 and starts sequence 1, so both sequences' chunk ranges turn invalid
    ws[260:264].view(torch.int32)[0] = 1 << 20      # seq_off[1]: far past the chunk table
    o = torch.full((B, T, H, 128), 7.0, dtype=torch.bfloat16, device=dev)
    hT = torch.full((4, H, 128, 128), 7.0, device=dev)
    kda.kda_fwd_inter(inp["h0"], inp["cu_seqlens"], o, hT, B=B, T=T, H=H, dk=128, dv=128,
                      dtype=torch.bfloat16, workspace=ws)
    code = kda.device_error()
    cu = inp["cu_seqlens"].tolist()
    untouched = bool((o[:, :cu[2]] == 7.0).all()) and bool((hT[:2] == 7.0).all())
    print("WORST", worst, "CODE", code, "UNTOUCHED", int(untouched), "AFTER", kda.device_error())
""") % ROOT


def test_debug_build_checks_pass_clean_runs_and_catch_a_corrupt_table():
    r = subprocess.run([sys.executable, "-c", DEBUG_CHILD], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    f = [x for x in r.stdout.splitlines() if x.startswith("WORST")][-1].split()
    assert float(f[1]) <= 1.0, f"debug build outside tolerance (worst / tol = {f[1]})"
    assert int(f[3]) == 10          # KDA_ERR_DEBUG_BOUNDS
    assert int(f[5]) == 1           # the refused sequences' outputs were not written
    assert int(f[7]) == 0           # read-and-clear
