"""The overlapped single-launch prefill through the C ABI: kda_fwd_overlapped, and
kda_fwd when its policy picks that schedule.

One launch holds both phases: state blocks walk each chain while prep workers in
the other blocks write the chunk records in time order and publish each through a
flag.  Parity is checked against the fp64 oracle at the bf16 tolerances of the
prefill (rel-L2 <= 1e-2, max-abs <= 5e-2), on ragged lengths (1 token, a partial
chunk, whole chunks, a ragged tail), with and without initial states, and at the
B=2, H=8, T=4,096 workload; against the two-launch schedule the results agree to
the same tolerance (the two slice the state differently, so their bf16 roundings
differ).
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


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def _close(got, ref, what, rel=1e-2, mx=5e-2):
    x = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(x).all(), f"{what}: non-finite values"
    r = float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))
    m = float(np.abs(x - ref).max()) if x.size else 0.0
    assert r <= rel and m <= mx, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"


def _oracle(inp):
    return oracle.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], None)


@pytest.mark.parametrize("B,T,H,h0", [(1, 1, 1, True), (2, 63, 3, False), (2, 64, 2, True),
                                      (2, 700, 3, True), (1, 4096, 4, False), (3, 1000, 5, True)])
def test_parity_with_oracle(B, T, H, h0):
    inp = W.make_prefill_inputs(B, T, H, 128, 128, torch.bfloat16, h0, seed=100 + T + H,
                                device=DEV)
    o, hT = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["h0"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    o_ref, hT_ref = _oracle(inp)
    _close(o, o_ref, "o")
    _close(hT, hT_ref, "hT")


def test_prefill_workload_and_two_launch_schedule():
    """B=2, H=8, T=4,096 (64 chunks per chain): the overlapped launch against the
    oracle on every token and head, and against the two launches."""
    inp = W.make_workload(W.PREFILL, DEV)
    o1, h1 = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                    inp["h0"])
    o2, h2 = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["h0"], num_segments=1)
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    o_ref, hT_ref = _oracle(inp)
    _close(o1, o_ref, "overlapped o")
    _close(h1, hT_ref, "overlapped hT")
    _close(o1, o2.double().cpu().numpy(), "overlapped vs two launches, o")
    _close(h1, h2.double().cpu().numpy(), "overlapped vs two launches, hT")


def test_policy_and_kda_fwd_dispatch():
    """kda_fwd takes the single launch for few long chains on a B200-sized GPU and
    then equals kda_fwd_overlapped bit for bit; packed input and many chains keep
    the two launches."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    bf = torch.bfloat16
    assert not kda.plan_overlap(1, 4096, 8, 128, 128, 3, bf)        # packed
    assert not kda.plan_overlap(8, 4096, 32, 128, 128, 0, bf)       # 256 chains
    assert not kda.plan_overlap(2, 4096, 8, 64, 64, 0, torch.float32)
    if sms < 128:
        pytest.skip("policy thresholds are for B200-sized GPUs")
    assert not kda.plan_overlap(2, 4096, 8, 128, 128, 0, bf)      # 64 chunks: too short
    assert kda.plan_overlap(2, 8192, 8, 128, 128, 0, bf)
    assert kda.plan_overlap(1, 1 << 20, 16, 128, 128, 0, bf)
    inp = W.make_prefill_inputs(2, 8192, 8, 128, 128, bf, True, seed=131, device=DEV)
    a = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    b = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    c = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(b[0], c[0]) and torch.equal(b[1], c[1])     # deterministic
    # no final state requested
    o, hT = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                        output_final_state=False)
    torch.cuda.synchronize()
    assert hT is None and torch.equal(o, a[0])


def test_checkpoints_on_the_overlapped_schedule():
    """kda_fwd_checkpointed where kda_fwd overlaps: o and hT equal kda_fwd's, and
    every stored state matches the oracle's state after that prefix."""
    bf = torch.bfloat16
    B, T, H, every = 2, 8192, 8, 2048
    if not kda.plan_overlap(B, T, H, 128, 128, 0, bf):
        pytest.skip("kda_fwd does not overlap at these sizes on this GPU")
    inp = W.make_prefill_inputs(B, T, H, 128, 128, bf, True, seed=132, device=DEV)
    o, hT, ck = kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                         inp["h0"], ckpt_every=every)
    o2, h2 = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    torch.cuda.synchronize()
    assert kda.device_error() == 0
    assert torch.equal(o, o2) and torch.equal(hT, h2)
    per = T // every
    assert ck.shape[0] == B * per
    for c in range(per):
        t = (c + 1) * every
        sub = {n: inp[n][:, :t] for n in ("q", "k", "v", "g", "beta")}
        sub["h0"] = inp["h0"]
        _, s_ref = _oracle(sub)
        for b in range(B):
            _close(ck[b * per + c], s_ref[b], f"checkpoint {c} of sequence {b}")


def test_in_place_state_update():
    """hT == h0 (the one allowed overlap): every state block reads its slice of h0
    before it writes hT."""
    inp = W.make_prefill_inputs(2, 700, 3, 128, 128, torch.bfloat16, True, seed=135, device=DEV)
    o_ref, hT_ref = _oracle(inp)
    S = inp["h0"].clone()
    o, hT = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S, hT=S)
    torch.cuda.synchronize()
    assert hT.data_ptr() == S.data_ptr()
    _close(o, o_ref, "o")
    _close(S, hT_ref, "hT in place")


def test_rejects_too_many_chains():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = sms // 2 + 1   # 2 * B * H >= SMs with B = 1
    inp = W.make_prefill_inputs(1, 64, H, 128, 128, torch.bfloat16, False, seed=133, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None)
    assert e.value.code == 2   # KDA_ERR_UNSUPPORTED_SHAPE


CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, %r)
    import kimi_delta_attention_28_b200 as kda
    from kimi_delta_attention_28_b200 import workloads as W
    inp = W.make_prefill_inputs(2, 512, 3, 128, 128, torch.bfloat16, True, seed=134,
                                device="cuda:0")
    o, hT = kda.kda_fwd_overlapped(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["h0"])
    code = kda.device_error()
    o2, _ = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  inp["h0"], num_segments=1)
    torch.cuda.synchronize()
    print("CODE", code, "AFTER", kda.device_error())
""") % ROOT


def test_bounded_wait_in_the_overlapped_launch():
    """With the state pass's first copy dropped (test hook), the state blocks' bounded
    waits run out, the call reports KDA_ERR_DEVICE_TIMEOUT, and the context stays
    usable for the next call (which reports its own, also timed-out, status: the hook
    applies to every state pass in the process)."""
    env = dict(os.environ, KDA_TEST_DROP_FIRST_COPY="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("CODE")][-1].split()
    assert int(line[1]) == 6          # KDA_ERR_DEVICE_TIMEOUT
    assert int(line[3]) == 6          # the second call's pass timed out the same way
