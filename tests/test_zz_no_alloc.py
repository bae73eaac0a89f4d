"""The allocation-free prefill entry point, kda_fwd_noalloc, called through the C ABI.

It exists for callers that cannot allocate device memory when they call the
library (for instance code that a host framework hands only its input and output
buffers, or code with a fixed memory budget where a per-call allocation is not
allowed).  Instead of a caller-provided workspace it uses a fixed 32 MiB scratch
array built into the library.  These checks run it twice in a row, on different
inputs, and compare each result with the regular workspace-based prefill run
without a time split (kda_fwd_segmented with one segment, the schedule the
allocation-free variant always uses): the same kernels on the same inputs, so the
results must agree bit for bit.  The second call also shows that what the first
call left in the shared array does not leak into the next result.  This file is
named so pytest collects it last.
"""
import pytest
import torch

import kimi_delta_attention_28_b200 as kda
from kimi_delta_attention_28_b200 import _lib
from kimi_delta_attention_28_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _same(got, ref, what):
    assert torch.equal(got, ref), (
        f"{what}: differs from the workspace entry point "
        f"(max-abs {float((got.double() - ref.double()).abs().max()):.3e})")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda.load_library()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [
        W.make_prefill_inputs(2, 700, 3, 128, 128, torch.bfloat16, True, seed=21, device=DEV),
        W.make_prefill_inputs(1, 0, 4, 128, 128, torch.bfloat16, True, seed=22, device=DEV,
                              lengths=[300, 0, 65, 1000]),
    ]
    for i, inp in enumerate(cases):
        assert _lib.workspace_size(*inp["q"].shape[:3], 128, 128,
                                   0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1,
                                   torch.bfloat16) <= _lib.NOALLOC_SCRATCH_BYTES
        o_ref, hT_ref = kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"],
                                              inp["beta"], inp["h0"], inp["cu_seqlens"],
                                              num_segments=1)
        o = torch.empty_like(o_ref)
        hT = torch.empty_like(hT_ref)
        kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                            inp["cu_seqlens"], o, hT)
        torch.cuda.synchronize()
        assert kda.device_error() == 0
        _same(o, o_ref, f"call {i + 1} o")
        _same(hT, hT_ref, f"call {i + 1} hT")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 57 chunks x 8 heads of 98,816-byte records exceed the 32 MiB array
    inp = W.make_prefill_inputs(1, 57 * 64, 8, 128, 128, torch.bfloat16, False, seed=23,
                                device=DEV)
    o = torch.full((1, 57 * 64, 8, 128), 3.0, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None, o,
                            None)
    assert e.value.code == 8
    torch.cuda.synchronize()
    assert bool((o == 3.0).all())      # nothing was launched
