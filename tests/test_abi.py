"""The C-ABI library builds, loads and exports every symbol ``include/kda.h``
declares; host-side argument validation answers with the documented status
codes.  CPU only: every call here returns before any kernel launch."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_28_b200 as kda
from kimi_delta_attention_28_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WS_SMALL = 0, 1, 2, 3, 4
BF16, F32 = 1, 0


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("kda_fwd", "kda_decode_step", "kda_fwd_workspace_size", "kda_fwd_intra",
              "kda_fwd_inter", "kda_get_last_device_error", "kda_status_string", "kda_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks a signature for {name}"


def test_binding_declares_nothing_extra():
    assert set(_lib.SIGNATURES) == set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.kda_version() >= 100
    for code in range(10):
        s = lib.kda_status_string(code).decode()
        assert s.startswith("KDA_")
    assert lib.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"


def test_workspace_size(lib):
    ws = lib.kda_fwd_workspace_size
    # tensor-core path stores one 98,816-byte record and one 4-byte ready flag (the
    # overlapped schedule's) per (64-token chunk, head)
    a = ws(2, 4096, 8, 128, 128, 0, BF16)
    b = ws(2, 4096 + 64, 8, 128, 128, 0, BF16)
    assert b - a == 2 * 8 * (98816 + 4)
    assert ws(1, 100, 4, 128, 128, 3, BF16) > 0          # packed varlen
    assert ws(2, 100, 4, 128, 128, 3, BF16) == 0         # packed needs B == 1
    assert ws(1, 64, 4, 128, 64, 0, BF16) == 0           # d_k != d_v
    assert ws(1, 64, 4, 96, 96, 0, BF16) == 0            # unsupported head size
    assert ws(1, 64, 4, 128, 128, 0, 7) == 0             # bad dtype
    assert 0 < ws(1, 64, 4, 32, 32, 0, F32) < 4096       # CUDA-core path: header only


def test_plan_segments_validates(lib):
    plan = lib.kda_fwd_plan_segments
    assert plan(1, 65536, 1, 128, 128, 0, BF16) >= 1     # 1 without a device
    assert plan(2, 4096, 8, 64, 64, 0, F32) == 1           # CUDA-core path never splits
    assert plan(2, 100, 4, 128, 64, 0, BF16) == 0          # d_k != d_v
    assert plan(2, 100, 4, 128, 128, 3, BF16) == 0         # packed needs B == 1


def test_plan_overlap_and_overlapped_validation(lib):
    plan = lib.kda_fwd_plan_overlap
    assert plan(2, 4096, 8, 128, 128, 0, BF16) == 0       # no device here
    assert plan(1, 4096, 8, 128, 128, 3, BF16) == 0       # packed input: never
    assert plan(2, 4096, 8, 64, 64, 0, F32) == 0          # CUDA-core path: never
    ov = lib.kda_fwd_overlapped
    p = 0x10000

    def call(**over):
        a = dict(q=p, k=p, v=p, g=p, beta=p, h0=None, B=2, T=128, H=2, dk=128, dv=128,
                 dtype=BF16, o=p + 0x100000, hT=None, work=p, ws=1 << 40, stream=None)
        a.update(over)
        return ov(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"], a["B"], a["T"], a["H"],
                  a["dk"], a["dv"], a["dtype"], a["o"], a["hT"], a["work"], a["ws"],
                  a["stream"])
    assert call(dk=64, dv=64) == UNSUPPORTED              # tensor-core path only
    assert call(dtype=F32) == UNSUPPORTED
    assert call(q=None) == INVALID
    assert call(B=-1) == INVALID
    assert call(q=p + 2) == MISALIGNED
    assert call(ws=1000) == WS_SMALL
    assert call() == 5                                    # KDA_ERR_CUDA: no device here


def test_segmented_workspace_size(lib):
    seg = lib.kda_fwd_segmented_workspace_size
    ws = lib.kda_fwd_workspace_size
    unit = 128 * 128 * 4 * 3                               # s_in (D x D) + seg_map (D x 2D), fp32
    # one segment: records only; the chain count (16) is too high for the split policy
    assert seg(2, 4096, 8, 128, 128, 0, BF16, 1) == ws(2, 4096, 8, 128, 128, 0, BF16)
    base = seg(1, 65536, 1, 128, 128, 0, BF16, 1)
    for n in (2, 5, 32):
        extra = seg(1, 65536, 1, 128, 128, 0, BF16, n) - base
        assert unit * n <= extra < unit * n + 512
    # the policy sizes for a 192-SM bound: 192 / (1 chain * 8 map tiles) = 24 segments
    assert ws(1, 65536, 1, 128, 128, 0, BF16) == seg(1, 65536, 1, 128, 128, 0, BF16, 24)
    # ... but never below 16 chunks per segment: 2048 tokens = 32 chunks -> 2 segments
    assert ws(1, 2048, 1, 128, 128, 0, BF16) == seg(1, 2048, 1, 128, 128, 0, BF16, 2)
    assert ws(1, 1024, 1, 128, 128, 0, BF16) == seg(1, 1024, 1, 128, 128, 0, BF16, 1)
    assert seg(1, 100, 1, 128, 128, 0, BF16, 0) == 0      # bad counts
    assert seg(1, 100, 1, 128, 128, 0, BF16, 4097) == 0
    assert seg(1, 100, 1, 64, 64, 0, F32, 2) == 0         # split needs the tensor-core path
    assert seg(1, 100, 1, 64, 64, 0, F32, 1) == ws(1, 100, 1, 64, 64, 0, F32)


def test_bwd_workspace_and_plan(lib):
    """kda_bwd's schedule: segments of whole chunks for bf16, d = 128, fixed-length
    input (one chunk each while (sequences x heads x segments) <= 1024, else the fewest
    power-of-two chunks that keep it so), the per-chain pass otherwise."""
    ws, seg, plan = (lib.kda_bwd_workspace_size, lib.kda_bwd_segmented_workspace_size,
                     lib.kda_bwd_plan_segments)
    assert plan(2, 4096, 8, 128, 128, 0, BF16) == 64        # 16 chains x 64 chunks
    assert plan(2, 8192, 8, 128, 128, 0, BF16) == 64        # 2 chunks per segment
    assert plan(1, 1 << 20, 16, 128, 128, 0, BF16) == 64    # 256 chunks per segment
    assert plan(3, 1000, 3, 128, 128, 0, BF16) == 16
    assert plan(1, 64, 2, 128, 128, 0, BF16) == 1           # one chunk: nothing to cut
    assert plan(2, 4096, 8, 64, 64, 0, F32) == 1            # CUDA-core path
    assert plan(1, 300, 2, 128, 128, 2, BF16) == 1          # packed
    assert plan(1, 100, 2, 128, 96, 0, BF16) == 0           # invalid sizes
    # the policy's workspace is the larger of the two schedules'
    assert ws(2, 4096, 8, 128, 128, 0, BF16) == seg(2, 4096, 8, 128, 128, 0, BF16, 64)
    assert seg(2, 4096, 8, 128, 128, 0, BF16, 0) == ws(2, 4096, 8, 128, 128, 0, BF16)
    one = seg(2, 4096, 8, 128, 128, 0, BF16, 1)
    assert 0 < one < seg(2, 4096, 8, 128, 128, 0, BF16, 2) < seg(2, 4096, 8, 128, 128, 0, BF16, 64)
    # per-unit scratch: 8 states of 128 x 128 fp32 per (sequence, head, segment)
    unit = 8 * 128 * 128 * 4
    d = seg(2, 4096, 8, 128, 128, 0, BF16, 64) - seg(2, 4096, 8, 128, 128, 0, BF16, 32)
    states = 2 * 2 * 32 * 8 * 128 * 128 * 4                 # start states and end gradients
    assert unit * 16 * 32 + states <= d < unit * 16 * 32 + states + 1024
    for n in (3, 128, -1):                                  # n must divide the 64 chunks
        assert seg(2, 4096, 8, 128, 128, 0, BF16, n) == 0
    assert seg(2, 4096, 8, 64, 64, 0, F32, 2) == 0
    assert seg(2, 4096, 8, 64, 64, 0, F32, 1) == ws(2, 4096, 8, 64, 64, 0, F32)
    assert seg(1, 300, 2, 128, 128, 2, BF16, 2) == 0        # packed: per-chain only


def _bwd(lib, nseg, ptr=0x10000, ws=1 << 40, **over):
    a = dict(q=ptr, k=ptr, v=ptr, g=ptr, beta=ptr, h0=None, cu=None, num_seqs=0, B=1, T=512,
             H=2, dk=128, dv=128, dtype=BF16, do=ptr, dhT=None, dq=0x200000, dk_=0x300000,
             dv_=0x400000, dg=0x500000, db=0x600000, dh0=None, work=0x700000, ws=ws,
             stream=None)
    a.update(over)
    return lib.kda_bwd_segmented(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"], a["cu"],
                                 a["num_seqs"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                 a["dtype"], a["do"], a["dhT"], a["dq"], a["dk_"], a["dv_"],
                                 a["dg"], a["db"], a["dh0"], nseg, a["work"], a["ws"],
                                 a["stream"])


def test_bwd_segmented_validation_before_launch(lib):
    assert _bwd(lib, -1) == INVALID
    assert _bwd(lib, 3) == UNSUPPORTED                       # 3 does not divide 8 chunks
    assert _bwd(lib, 16) == UNSUPPORTED
    assert _bwd(lib, 2, dk=64, dv=64, dtype=F32) == UNSUPPORTED
    assert _bwd(lib, 2, cu=0x30000, num_seqs=2, B=1) == UNSUPPORTED
    assert _bwd(lib, 2, do=0x10002) == MISALIGNED            # 16-byte vector reads of dO
    assert _bwd(lib, 1, do=0x10008) == MISALIGNED            # every schedule stages dO rows
    assert _bwd(lib, 1, g=0x10008, dtype=F32, dk=64, dv=64) == MISALIGNED   # ... and g rows
    assert _bwd(lib, 2, dq=0x200002) == MISALIGNED
    assert _bwd(lib, 2, dk_=0x300008) == MISALIGNED
    assert _bwd(lib, 2, ws=1024) == WS_SMALL
    assert _bwd(lib, 2, dq=0x10000) == INVALID               # a gradient aliases an input


def _fwd(lib, ptr=0x10000, ws=1 << 40, **over):
    a = dict(q=ptr, k=ptr, v=ptr, g=ptr, beta=ptr, h0=None, cu=None, num_seqs=0, B=1, T=64,
             H=2, dk=128, dv=128, dtype=BF16, o=ptr + 0x100000, hT=None, work=ptr, ws=ws,
             stream=None)
    a.update(over)
    return lib.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"], a["cu"],
                       a["num_seqs"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["dtype"],
                       a["o"], a["hT"], a["work"], a["ws"], a["stream"])


def test_fwd_validation_before_launch(lib):
    assert _fwd(lib, dtype=5) == INVALID
    assert _fwd(lib, dk=64, dv=128) == UNSUPPORTED
    assert _fwd(lib, dk=96, dv=96) == UNSUPPORTED
    assert _fwd(lib, H=0) == INVALID
    assert _fwd(lib, B=-1) == INVALID
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, o=None) == INVALID
    assert _fwd(lib, q=0x10004) == MISALIGNED
    assert _fwd(lib, hT=0x20008) == MISALIGNED           # states are read as float4
    assert _fwd(lib, g=0x10004) == MISALIGNED            # g is read as float pairs
    assert _fwd(lib, g=0x10008) == MISALIGNED            # ... and by tensor copies (bf16, d=128)
    assert _fwd(lib, g=0x10008, dtype=F32, dk=64, dv=64, B=0) == OK   # CUDA-core path: 8 bytes
    assert _fwd(lib, o=0x20002) == MISALIGNED            # bf16 o needs 4 bytes
    assert _fwd(lib, o=0x10000) == INVALID               # output aliases an input
    assert _fwd(lib, ws=16) == WS_SMALL
    assert _fwd(lib, work=None) == WS_SMALL
    assert _fwd(lib, num_seqs=2) == INVALID              # offsets count without offsets
    assert _fwd(lib, cu=0x30000, num_seqs=2, B=2) == INVALID   # packed needs B == 1
    assert _fwd(lib, cu=0x30002, num_seqs=2) == MISALIGNED
    # empty batch: valid, nothing to do, no launch
    assert _fwd(lib, B=0) == OK


def test_checkpointed_validation_before_launch(lib):
    """kda_fwd_checkpointed checks its checkpoint arguments on the host, before any
    launch: interval a positive multiple of 64, enough slots for fixed-length input,
    a 16-byte aligned buffer, the tensor-core path only."""
    p = 0x10000

    def ck(every=256, ckpts=0x40000, cap=2, B=1, T=512, H=2, dk=128, dtype=BF16, cu=None,
           num_seqs=0):
        return lib.kda_fwd_checkpointed(p, p, p, p, p, None, cu, num_seqs, B, T, H, dk, dk, dtype,
                                        p + 0x100000, None, every, ckpts, cap, p, 1 << 40, None)
    assert ck(every=100) == INVALID                     # not a chunk boundary
    assert ck(every=0) == INVALID
    assert ck(every=-64) == INVALID
    assert ck(cap=1) == INVALID                         # 512 // 256 = 2 checkpoints needed
    assert ck(B=3, cap=5) == INVALID                    # 3 sequences x 2
    assert ck(ckpts=None, cap=2) == INVALID             # slots promised, no buffer
    assert ck(cap=-1) == INVALID
    assert ck(ckpts=0x40008) == MISALIGNED              # stored as float4
    assert ck(dk=64) == UNSUPPORTED                     # tensor-core path only
    assert ck(dtype=F32) == UNSUPPORTED
    assert ck(B=0) == OK                                # nothing to do, no launch
    assert lib.kda_status_string(9).decode().startswith("KDA_ERR_CHECKPOINT_CAPACITY")


def test_checkpoint_count():
    """Slots kda_fwd_checkpointed needs: the sum over sequences of length // interval."""
    import torch
    assert kda.checkpoint_count(1000, 128, B=2) == 2 * 7
    assert kda.checkpoint_count(63, 64, B=4) == 0
    cu = torch.tensor([0, 300, 300, 1000, 1064, 1193], dtype=torch.int32)   # 300, 0, 700, 64, 129
    assert kda.checkpoint_count(1193, 64, cu_seqlens=cu) == 4 + 0 + 10 + 1 + 2
    assert kda.checkpoint_count(1193, 256, cu_seqlens=cu) == 1 + 0 + 2 + 0 + 0


def test_phase_entry_points_validate(lib):
    p = 0x10000
    assert lib.kda_fwd_intra(p, p, p, p, p, None, 0, 1, 64, 2, 32, 32, F32, p, 1 << 40,
                             None) == UNSUPPORTED
    assert lib.kda_fwd_inter(None, None, 0, 1, 64, 2, 128, 128, BF16, None, None, p, 1 << 40,
                             None) == INVALID
    assert lib.kda_fwd_inter(None, None, 0, 0, 64, 2, 128, 128, BF16, p, None, p, 1 << 40,
                             None) == OK


def test_decode_validation_before_launch(lib):
    p = 0x10000
    f = lib.kda_decode_step
    assert f(p, p, p, p, p, p, p, 4, 2, 128, 64, BF16, None) == UNSUPPORTED
    assert f(p, p, p, p, p, p, p, 4, 2, 128, 128, 9, None) == INVALID
    assert f(p, p, p, p, p, None, p, 4, 2, 128, 128, BF16, None) == INVALID
    assert f(p, p, p, p, p, p + 8, p, 4, 2, 128, 128, BF16, None) == MISALIGNED
    assert f(p, p, p, p, p + 2, p, p, 4, 2, 128, 128, BF16, None) == MISALIGNED
    assert f(p, p, p, p, p, p, p, 0, 2, 128, 128, BF16, None) == OK
    assert f(p, p, p, p, p, p, p, -1, 2, 128, 128, BF16, None) == INVALID


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kda.kda_fwd(x, x, x, x.float(), torch.zeros(1, 4, 1), None)


def test_python_binding_checks_shapes_before_launch():
    """The C ABI sees raw pointers, so the binding checks every tensor's shape
    against q's (metadata only: these CPU tensors never reach the library)."""
    import torch
    B, T, H, d = 1, 8, 2, 64
    q = torch.zeros(B, T, H, d, dtype=torch.bfloat16)
    g = torch.zeros(B, T, H, d)
    beta = torch.zeros(B, T, H)
    short = torch.zeros(B, T - 1, H, d, dtype=torch.bfloat16)
    cases = [
        dict(k=short), dict(v=short), dict(g=g[:, :-1]), dict(beta=beta[:, :-1]),
        dict(h0=torch.zeros(B, H, d, d - 1)), dict(o=short),
        dict(hT=torch.zeros(B + 1, H, d, d)),
        dict(workspace=torch.zeros(16, dtype=torch.float32)),
        dict(cu_seqlens=torch.tensor([0, 4, 8], dtype=torch.int32), h0=torch.zeros(1, H, d, d)),
    ]
    for over in cases:
        a = dict(q=q, k=q, v=q, g=g, beta=beta, h0=None)
        a.update(over)
        kw = {n: a.pop(n) for n in ("o", "hT", "workspace", "cu_seqlens") if n in a}
        cu = kw.pop("cu_seqlens", None)
        with pytest.raises(ValueError, match="shape|workspace|cu_seqlens"):
            kda.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["h0"], cu, **kw)
    with pytest.raises(ValueError, match="shape"):   # decode: state of the wrong size
        kda.kda_decode_step(q[0], q[0], q[0], g[0], beta[0], torch.zeros(T, H, d, d + 1))
    with pytest.raises(ValueError, match="B == 1"):
        kda.kda_fwd(q.expand(2, T, H, d), q.expand(2, T, H, d), q.expand(2, T, H, d),
                    g.expand(2, T, H, d), beta.expand(2, T, H), None,
                    torch.tensor([0, 8], dtype=torch.int32))


def test_library_is_built_for_sm100a():
    # the build recipe targets sm_100a only
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)
    assert os.path.exists(build.LIB)
    ctypes.CDLL(build.LIB)
