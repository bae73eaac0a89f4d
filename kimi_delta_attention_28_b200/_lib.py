"""ctypes binding of ``libkda_b200.so`` (the C ABI in ``include/kda.h``).

Argument marshalling only: every step of the recurrence runs in the library's
CUDA kernels.  torch provides device memory (outputs, workspace) and the
current CUDA stream.  If the library is missing the calls raise; there is no
other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda_b200.so")
# The same library built with device-side bounds checks (-DKDA_DEBUG=1); load it with
# load_library(DEBUG_LIB_PATH) before any other call.
DEBUG_LIB_PATH = os.path.join(HERE, "libkda_b200_debug.so")

KDA_DTYPE_F32 = 0
KDA_DTYPE_BF16 = 1

STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED_SHAPE",
          3: "KDA_ERR_MISALIGNED", 4: "KDA_ERR_WORKSPACE_TOO_SMALL", 5: "KDA_ERR_CUDA",
          6: "KDA_ERR_DEVICE_TIMEOUT", 7: "KDA_ERR_BAD_SEQLENS",
          8: "KDA_ERR_EXCEEDS_STATIC_SCRATCH", 9: "KDA_ERR_CHECKPOINT_CAPACITY",
          10: "KDA_ERR_DEBUG_BOUNDS", 11: "KDA_ERR_BAD_ACCEPTED"}

# Largest number of drafted tokens kda_decode_verify / kda_decode_commit take.
MAX_DRAFT = 16

# Size of the static scratch array behind kda_fwd_noalloc (KDA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 32 << 20

# Every symbol the header declares, with its ctypes signature.
_VP, _SZ, _I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "kda_version": ([], _I),
    "kda_build_flags": ([], _I),
    "kda_status_string": ([_I], ctypes.c_char_p),
    "kda_fwd_workspace_size": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "kda_fwd": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP,
                 _SZ, _VP], _I),
    "kda_fwd_intra": ([_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _SZ, _VP],
                      _I),
    "kda_fwd_inter": ([_VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP], _I),
    "kda_decode_step": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _VP], _I),
    "kda_get_last_device_error": ([_VP], _I),
    "kda_cp_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "kda_cp_local_map": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _SZ, _VP],
                         _I),
    "kda_cp_finish": ([_VP, _I, _I, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP],
                      _I),
    "kda_bwd_workspace_size": ([_I, _I, _I, _I, _I, _I, _I], _SZ),
    "kda_bwd": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP,
                 _VP, _VP, _VP, _VP, _VP, _SZ, _VP], _I),
    "kda_bwd_segmented_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _I], _SZ),
    "kda_bwd_plan_segments": ([_I, _I, _I, _I, _I, _I, _I], _I),
    "kda_bwd_segmented": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _VP,
                           _VP, _VP, _VP, _VP, _VP, _VP, _I, _VP, _SZ, _VP], _I),
    "kda_decode_verify": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP], _I),
    "kda_decode_commit": ([_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP], _I),
    "kda_fwd_noalloc": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _VP,
                         _VP], _I),
    "kda_fwd_overlapped": ([_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _VP,
                            _SZ, _VP], _I),
    "kda_fwd_plan_overlap": ([_I, _I, _I, _I, _I, _I, _I], _I),
    "kda_fwd_segmented_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _I], _SZ),
    "kda_fwd_plan_segments": ([_I, _I, _I, _I, _I, _I, _I], _I),
    "kda_fwd_segmented": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I,
                           _VP, _VP, _VP, _SZ, _VP], _I),
    "kda_fwd_checkpointed": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP,
                              _VP, _I, _VP, ctypes.c_longlong, _VP, _SZ, _VP], _I),
}


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({_status_string(code)})")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (built by ``kimi_delta_attention_28_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m kimi_delta_attention_28_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _status_string(code: int) -> str:
    try:
        return load_library().kda_status_string(code).decode()
    except Exception:  # noqa: BLE001 - only used to decorate an error message
        return "?"


def _check(code: int, where: str):
    if code != 0:
        raise KDAError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return KDA_DTYPE_BF16
    if dt == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {dt}")


def _need(t, name, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _shape(t, name, shape):
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _prefill_shapes(q, k, v, g, beta, h0=None, cu_seqlens=None, o=None, hT=None,
                    workspace=None):
    """Check the tensors' shapes against q's [B, T, H, d_k] (metadata only; the C ABI
    sees raw pointers and would read past a short tensor).  Returns (B, T, H, dk, dv,
    num_seqs, N)."""
    if q.dim() != 4:
        raise ValueError(f"q must be [B, T, H, d_k], got shape {tuple(q.shape)}")
    B, T, H, dk = q.shape
    if v.dim() != 4 or tuple(v.shape[:3]) != (B, T, H):
        raise ValueError(f"v has shape {tuple(v.shape)}, expected ({B}, {T}, {H}, d_v)")
    dv = v.shape[3]
    _shape(k, "k", q.shape)
    _shape(g, "g", q.shape)
    _shape(beta, "beta", (B, T, H))
    num_seqs = 0
    if cu_seqlens is not None:
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be a 1-D tensor of N + 1 offsets")
        if B != 1:
            raise ValueError("packed sequences (cu_seqlens) need B == 1")
        num_seqs = cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    _shape(h0, "h0", (N, H, dk, dv))
    _shape(o, "o", (B, T, H, dv))
    _shape(hT, "hT", (N, H, dk, dv))
    if workspace is not None and (workspace.dtype != torch.uint8 or workspace.dim() != 1):
        raise ValueError("workspace must be a 1-D uint8 tensor (its numel is the byte count)")
    return B, T, H, dk, dv, num_seqs, N


def workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                   dtype: torch.dtype) -> int:
    return int(load_library().kda_fwd_workspace_size(B, T, H, dk, dv, num_seqs,
                                                      _dtype_code(dtype)))


def kda_fwd(q, k, v, g, beta, h0=None, cu_seqlens=None, *, output_final_state: bool = True,
            o=None, hT=None, workspace=None):
    """Chunkwise KDA prefill through the C ABI.

    q, k, g: [B, T, H, d_k]; v: [B, T, H, d_v] (q/k/v bf16 or fp32, g fp32);
    beta: [B, T, H] fp32; h0: [N, H, d_k, d_v] fp32 or None (zeros);
    cu_seqlens: int32 [N+1] packed offsets (then B == 1) or None.
    Returns (o, hT); hT is None when output_final_state is False.
    """
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(q, k, v, g, beta, h0, cu_seqlens, o, hT,
                                                   workspace)
    dt = _dtype_code(q.dtype)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    if hT is None and output_final_state:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    need = workspace_size(B, T, H, dk, dv, num_seqs, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.kda_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                       _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, dt, _ptr(o), _ptr(hT),
                       _ptr(workspace), workspace.numel(), _stream(dev)), "kda_fwd")
    return o, hT


def segmented_workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                             dtype: torch.dtype, num_segments: int) -> int:
    return int(load_library().kda_fwd_segmented_workspace_size(
        B, T, H, dk, dv, num_seqs, _dtype_code(dtype), num_segments))


def plan_segments(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                  dtype: torch.dtype) -> int:
    """Time segments kda_fwd uses for these sizes on the current device (1: none)."""
    return int(load_library().kda_fwd_plan_segments(B, T, H, dk, dv, num_seqs,
                                                    _dtype_code(dtype)))


def kda_fwd_segmented(q, k, v, g, beta, h0=None, cu_seqlens=None, *, num_segments: int,
                      o=None, hT=None, workspace=None):
    """kda_fwd with the state pass split into ``num_segments`` time segments per
    (sequence, head) chain (segment maps, a sequential combine, then the output
    pass from each segment's starting state).  Arguments as for kda_fwd; always
    returns (o, hT)."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(q, k, v, g, beta, h0, cu_seqlens, o, hT,
                                                   workspace)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    if hT is None:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    need = segmented_workspace_size(B, T, H, dk, dv, num_seqs, q.dtype, num_segments)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.kda_fwd_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                 _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv,
                                 _dtype_code(q.dtype), num_segments, _ptr(o), _ptr(hT),
                                 _ptr(workspace), workspace.numel(), _stream(dev)),
           "kda_fwd_segmented")
    return o, hT


def plan_overlap(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                 dtype: torch.dtype) -> bool:
    """Whether kda_fwd runs both phases as one overlapped launch for these sizes."""
    return bool(load_library().kda_fwd_plan_overlap(B, T, H, dk, dv, num_seqs,
                                                    _dtype_code(dtype)))


def kda_fwd_overlapped(q, k, v, g, beta, h0=None, *, o=None, hT=None, workspace=None):
    """Fixed-length prefill with the record and state phases in one launch (the
    state blocks consume each chunk record as soon as it is published).  Needs
    2 * B * H below the SM count.  Arguments as for kda_fwd; returns (o, hT)."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(q, k, v, g, beta, h0, None, o, hT,
                                                   workspace)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    if hT is None:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    need = segmented_workspace_size(B, T, H, dk, dv, 0, q.dtype, 1)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.kda_fwd_overlapped(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                  B, T, H, dk, dv, _dtype_code(q.dtype), _ptr(o), _ptr(hT),
                                  _ptr(workspace), workspace.numel(), _stream(dev)),
           "kda_fwd_overlapped")
    return o, hT


def checkpoint_count(T: int, ckpt_every: int, B: int = 1, cu_seqlens=None) -> int:
    """Number of state checkpoints kda_fwd_checkpointed stores per head: sum over the
    sequences of length // ckpt_every (reads packed lengths back from the device)."""
    if cu_seqlens is None:
        return B * (T // ckpt_every)
    lens = (cu_seqlens[1:] - cu_seqlens[:-1]).to("cpu", torch.int64)
    return int((lens // ckpt_every).sum())


def kda_fwd_checkpointed(q, k, v, g, beta, h0=None, cu_seqlens=None, *, ckpt_every: int = 256,
                         ckpts=None, o=None, hT=None, workspace=None):
    """kda_fwd that also stores the state after every ``ckpt_every`` tokens of each
    sequence (a multiple of 64), for prefix caching.  Returns (o, hT, ckpts) with
    ckpts [num_checkpoints, H, d_k, d_v] fp32: each sequence's checkpoints together, in
    token order; checkpoint c of a sequence is its state after (c + 1) * ckpt_every
    tokens.  When ``ckpts`` is not given it is allocated here (packed input: the
    lengths are read back from the device)."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(q, k, v, g, beta, h0, cu_seqlens, o, hT,
                                                   workspace)
    if ckpt_every <= 0 or ckpt_every % 64:
        raise ValueError(f"ckpt_every must be a positive multiple of 64, got {ckpt_every}")
    if ckpts is not None and (ckpts.dim() != 4 or tuple(ckpts.shape[1:]) != (H, dk, dv)):
        raise ValueError(f"ckpts has shape {tuple(ckpts.shape)}, expected (n, {H}, {dk}, {dv})")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(ckpts, "ckpts", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    if ckpts is None:
        ckpts = torch.empty(checkpoint_count(T, ckpt_every, B, cu_seqlens), H, dk, dv,
                            dtype=torch.float32, device=dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    if hT is None:
        hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    need = workspace_size(B, T, H, dk, dv, num_seqs, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.kda_fwd_checkpointed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                    _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv,
                                    _dtype_code(q.dtype), _ptr(o), _ptr(hT), ckpt_every,
                                    _ptr(ckpts) if ckpts.numel() else None, ckpts.shape[0],
                                    _ptr(workspace), workspace.numel(), _stream(dev)),
           "kda_fwd_checkpointed")
    return o, hT, ckpts


def kda_fwd_intra(q, k, v, g, beta, cu_seqlens=None, *, workspace):
    """Phase 1 of the tensor-core prefill (bf16, d = 128): per-(chunk, head)
    intra-chunk records into ``workspace``.  Same argument conventions as kda_fwd."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, _ = _prefill_shapes(q, k, v, g, beta, None, cu_seqlens,
                                                   workspace=workspace)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    _check(lib.kda_fwd_intra(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                             num_seqs, B, T, H, dk, dv, _dtype_code(q.dtype), _ptr(workspace),
                             workspace.numel(), _stream(dev)), "kda_fwd_intra")


def kda_fwd_inter(h0, cu_seqlens, o, hT, *, B, T, H, dk, dv, dtype, workspace):
    """Phase 2 of the tensor-core prefill: the state pass, writing o and hT."""
    lib = load_library()
    dev = o.device
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    _shape(o, "o", (B, T, H, dv))
    _shape(h0, "h0", (N, H, dk, dv))
    _shape(hT, "hT", (N, H, dk, dv))
    _need(o, "o", dtype, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    _check(lib.kda_fwd_inter(_ptr(h0), _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv,
                             _dtype_code(dtype), _ptr(o), _ptr(hT), _ptr(workspace),
                             workspace.numel(), _stream(dev)), "kda_fwd_inter")


def kda_decode_step(q, k, v, g, beta, S, o=None):
    """One decode token per (sequence, head); S [N, H, d_k, d_v] fp32 is updated
    in place.  q, k, g: [N, H, d_k]; v: [N, H, d_v]; beta: [N, H].  Returns o."""
    lib = load_library()
    dev = q.device
    if q.dim() != 3 or v.dim() != 3 or tuple(v.shape[:2]) != tuple(q.shape[:2]):
        raise ValueError(f"q must be [N, H, d_k] and v [N, H, d_v], got {tuple(q.shape)} "
                         f"and {tuple(v.shape)}")
    N, H, dk = q.shape
    dv = v.shape[-1]
    _shape(k, "k", q.shape)
    _shape(g, "g", q.shape)
    _shape(beta, "beta", (N, H))
    _shape(S, "S", (N, H, dk, dv))
    _shape(o, "o", (N, H, dv))
    dt = _dtype_code(q.dtype)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=dev)
    _check(lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                               N, H, dk, dv, dt, _stream(dev)), "kda_decode_step")
    return o


def cp_workspace_size(B: int, T_local: int, H: int, dk: int, dv: int,
                      dtype: torch.dtype) -> int:
    return int(load_library().kda_cp_workspace_size(B, T_local, H, dk, dv, _dtype_code(dtype)))


def kda_cp_local_map(q, k, v, g, beta, *, workspace):
    """Step 1 of context parallelism: the local stretch's map [R | P] per (sequence,
    head), fp32 [B, H, d_k, 2 d_v]; the chunk records stay in ``workspace``."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, _, _ = _prefill_shapes(q, k, v, g, beta, workspace=workspace)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    seg_map = torch.empty(B, H, dk, 2 * dv, dtype=torch.float32, device=dev)
    _check(lib.kda_cp_local_map(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), B, T, H, dk, dv,
                                _dtype_code(q.dtype), _ptr(seg_map), _ptr(workspace),
                                workspace.numel(), _stream(dev)), "kda_cp_local_map")
    return seg_map


def kda_cp_finish(maps, rank, h0, *, B, T_local, H, dk, dv, dtype, o, hT, workspace):
    """Step 3: fold the gathered maps [world, B, H, d_k, 2 d_v] of ranks before `rank`
    onto h0, then run the local state pass; writes o [B, T_local, H, d_v] and hT (the
    state after the local stretch).  Returns (o, hT, s_in)."""
    lib = load_library()
    dev = o.device
    world = maps.shape[0]
    _shape(maps, "maps", (world, B, H, dk, 2 * dv))
    _shape(h0, "h0", (B, H, dk, dv))
    _shape(o, "o", (B, T_local, H, dv))
    _shape(hT, "hT", (B, H, dk, dv))
    _need(maps, "maps", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(o, "o", dtype, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    s_in = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    _check(lib.kda_cp_finish(_ptr(maps), rank, world, _ptr(h0), _ptr(s_in), B, T_local, H, dk,
                             dv, _dtype_code(dtype), _ptr(o), _ptr(hT), _ptr(workspace),
                             workspace.numel(), _stream(dev)), "kda_cp_finish")
    return o, hT, s_in


def gather_segment_maps(seg_map, group=None):
    """Step 2: all-gather every rank's [R | P] in rank order -> [world, ...] (one
    collective through torch.distributed; NCCL on GPUs)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(seg_map) for _ in range(world)]
    dist.all_gather(parts, seg_map.contiguous(), group=group)
    return torch.stack(parts)


def kda_fwd_context_parallel(q, k, v, g, beta, h0=None, *, group=None, workspace=None):
    """Prefill of a batch split in time over the ranks of ``group``: this rank holds
    tokens [rank T_local, (rank + 1) T_local) of every sequence (q, k, v, g [B, T_local,
    H, d]; beta [B, T_local, H]); h0 [B, H, d_k, d_v] are the sequences' initial states
    (the same on every rank; None: zeros).  Returns this rank's outputs o and the state
    after its stretch (on the last rank: the final states)."""
    import torch.distributed as dist
    B, T, H, dk, dv, _, _ = _prefill_shapes(q, k, v, g, beta, h0, workspace=workspace)
    dev = q.device
    if workspace is None:
        workspace = torch.empty(max(cp_workspace_size(B, T, H, dk, dv, q.dtype), 256),
                                dtype=torch.uint8, device=dev)
    seg_map = kda_cp_local_map(q, k, v, g, beta, workspace=workspace)
    maps = gather_segment_maps(seg_map, group)
    rank = dist.get_rank(group)
    o = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    hT = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    kda_cp_finish(maps, rank, h0, B=B, T_local=T, H=H, dk=dk, dv=dv, dtype=q.dtype, o=o, hT=hT,
                  workspace=workspace)
    return o, hT


def bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                       dtype: torch.dtype) -> int:
    return int(load_library().kda_bwd_workspace_size(B, T, H, dk, dv, num_seqs,
                                                     _dtype_code(dtype)))


def bwd_segmented_workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                                 dtype: torch.dtype, num_segments: int) -> int:
    return int(load_library().kda_bwd_segmented_workspace_size(B, T, H, dk, dv, num_seqs,
                                                               _dtype_code(dtype), num_segments))


def bwd_plan_segments(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                      dtype: torch.dtype) -> int:
    """Segments per sequence kda_bwd uses (1: the per-chain pass)."""
    return int(load_library().kda_bwd_plan_segments(B, T, H, dk, dv, num_seqs, _dtype_code(dtype)))


def kda_bwd(q, k, v, g, beta, h0, cu_seqlens, grad_o, grad_hT=None, *, workspace=None):
    """Gradient of a loss through kda_fwd: given grad_o = dL/do [B, T, H, d_v] (dtype of
    q) and grad_hT = dL/dhT [N, H, d_k, d_v] fp32 (None: zero), returns (dq, dk, dv, dg,
    dbeta, dh0): dq, dk, dv in the dtype of q, the rest fp32 (dh0 None when h0 is None)."""
    return _bwd(q, k, v, g, beta, h0, cu_seqlens, grad_o, grad_hT, None, workspace)


def kda_bwd_segmented(q, k, v, g, beta, h0, cu_seqlens, grad_o, grad_hT=None, *,
                      num_segments: int, workspace=None):
    """kda_bwd with the schedule given: num_segments 0 as kda_bwd, 1 the per-chain pass,
    n >= 2 n segments per sequence (n divides ceil(T / 64); bf16, d = 128, fixed length)."""
    return _bwd(q, k, v, g, beta, h0, cu_seqlens, grad_o, grad_hT, int(num_segments), workspace)


def _bwd(q, k, v, g, beta, h0, cu_seqlens, grad_o, grad_hT, num_segments, workspace):
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, N = _prefill_shapes(q, k, v, g, beta, h0, cu_seqlens,
                                                   workspace=workspace)
    _shape(grad_o, "grad_o", (B, T, H, dv))
    _shape(grad_hT, "grad_hT", (N, H, dk, dv))
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (grad_o, "grad_o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(grad_hT, "grad_hT", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(workspace, "workspace", torch.uint8, dev)
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg, db = torch.empty_like(g), torch.empty_like(beta)
    dh0 = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev) if h0 is not None else None
    if num_segments is None:
        need = bwd_workspace_size(B, T, H, dk, dv, num_seqs, q.dtype)
    else:
        need = bwd_segmented_workspace_size(B, T, H, dk, dv, num_seqs, q.dtype, num_segments)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    common = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(cu_seqlens),
              num_seqs, B, T, H, dk, dv, _dtype_code(q.dtype), _ptr(grad_o), _ptr(grad_hT),
              _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(db), _ptr(dh0))
    if num_segments is None:
        _check(lib.kda_bwd(*common, _ptr(workspace), workspace.numel(), _stream(dev)), "kda_bwd")
    else:
        _check(lib.kda_bwd_segmented(*common, num_segments, _ptr(workspace), workspace.numel(),
                                     _stream(dev)), "kda_bwd_segmented")
    return dq, dk_, dv_, dg, db, dh0


def _draft_shapes(k, v, g, beta, S, q=None):
    if k.dim() != 4 or v.dim() != 4 or tuple(v.shape[:3]) != tuple(k.shape[:3]):
        raise ValueError(f"k must be [N, K, H, d_k] and v [N, K, H, d_v], got {tuple(k.shape)} "
                         f"and {tuple(v.shape)}")
    N, K, H, dk = k.shape
    dv = v.shape[-1]
    _shape(q, "q", k.shape)
    _shape(g, "g", k.shape)
    _shape(beta, "beta", (N, K, H))
    _shape(S, "S", (N, H, dk, dv))
    if K > MAX_DRAFT:
        raise ValueError(f"at most {MAX_DRAFT} drafted tokens, got K = {K}")
    return N, K, H, dk, dv


def kda_decode_verify(q, k, v, g, beta, S, o=None):
    """Run K drafted tokens per (sequence, head) from the state S without changing it.
    q, k, g: [N, K, H, d_k]; v: [N, K, H, d_v]; beta: [N, K, H]; S: [N, H, d_k, d_v]
    fp32.  Returns o [N, K, H, d_v]: o[:, t] is what the t-th of K chained decode steps
    would return."""
    lib = load_library()
    dev = k.device
    N, K, H, dk, dv = _draft_shapes(k, v, g, beta, S, q)
    _shape(o, "o", (N, K, H, dv))
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, k.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    if o is None:
        o = torch.empty(N, K, H, dv, dtype=k.dtype, device=dev)
    _check(lib.kda_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                 _ptr(o), N, K, H, dk, dv, _dtype_code(k.dtype), _stream(dev)),
           "kda_decode_verify")
    return o


def kda_decode_commit(k, v, g, beta, accepted, S):
    """Advance S in place over the first accepted[n] of the K drafted tokens of each
    sequence n (the inputs given to kda_decode_verify); accepted is an int32 CUDA
    tensor [N] with values in [0, K].  Returns S."""
    lib = load_library()
    dev = k.device
    N, K, H, dk, dv = _draft_shapes(k, v, g, beta, S)
    _shape(accepted, "accepted", (N,))
    for t, n in ((k, "k"), (v, "v")):
        _need(t, n, k.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(S, "S", torch.float32, dev)
    _need(accepted, "accepted", torch.int32, dev)
    _check(lib.kda_decode_commit(_ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(accepted), _ptr(S),
                                 N, K, H, dk, dv, _dtype_code(k.dtype), _stream(dev)),
           "kda_decode_commit")
    return S


def kda_fwd_noalloc(q, k, v, g, beta, h0, cu_seqlens, o, hT):
    """Prefill through the allocation-free entry point: the library uses its
    built-in static scratch array instead of a workspace.  For callers that
    cannot allocate device memory per call; the caller passes every buffer,
    including the outputs o and hT (hT may be None), and this wrapper allocates
    nothing.  bf16, d = 128 only; the problem must fit the 32 MiB scratch."""
    lib = load_library()
    dev = q.device
    B, T, H, dk, dv, num_seqs, _ = _prefill_shapes(q, k, v, g, beta, h0, cu_seqlens, o, hT)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(h0, "h0", torch.float32, dev)
    _need(hT, "hT", torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _check(lib.kda_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                               _ptr(cu_seqlens), num_seqs, B, T, H, dk, dv, _dtype_code(q.dtype),
                               _ptr(o), _ptr(hT), _stream(dev)), "kda_fwd_noalloc")
    return o, hT


def device_error(device=None) -> int:
    """Synchronise and read/clear the library's device error word (0 = none)."""
    dev = torch.device(device) if device is not None else torch.device("cuda")
    return int(load_library().kda_get_last_device_error(_stream(dev)))
