"""Python front end of the fp64 CPU oracle for the KDA recurrence.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may call this module; the product path never does.  It imports
nothing from the CUDA package.

The recurrence it evaluates is the single-head KDA update from the "Kimi K3"
open-weights field notes (ailearn.mscapital.top/kimi-k3.html), panel
"KDA 单头递归" (KDA single-head recurrence)::

    S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t

Inputs are widened to fp64 exactly (bf16 and fp32 values are representable in
fp64), so the oracle sees precisely the numbers a GPU kernel sees.

Parity status of each function (what pins it, beside itself, lives in
``tests/test_oracle_pins.py``):

* ``kda_fwd``          pinned: brute-force operator products (float and exact
                       rational), closed forms (beta=0 decay, last-write
                       retrieval, orthonormal-key memory, d_k=1 scalar form),
                       chunked evaluation at several chunk sizes, and
                       invariants (linearity, split runs, varlen).
* ``kda_decode_step``  pinned: equals ``kda_fwd`` with T=1 and chained decode
                       equals prefill.
* ``kda_bwd`` / ``kda_bwd_packed``  (the gradient of the recurrence, by reverse
                       accumulation through the token loop) pinned: against central
                       finite differences of ``kda_fwd`` in every input, element by
                       element on tiny chains and along random directions on larger
                       packed batches (empty sequences included); planted mistakes in
                       its C source fail those pins.
* ``kda_decode_verify`` / ``kda_decode_commit``  (speculative decoding, same page,
                       panel "目标模型太大，缓存和草稿都必须理解 KDA": the state must
                       follow only the accepted draft tokens) pinned: against the
                       brute-force operator products on every drafted prefix, with
                       a different accepted count per sequence, and commit of zero
                       tokens returns the state unchanged.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, lp,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int, dp, dp]
        lib.kda_oracle_fwd.restype = ctypes.c_int
        lib.kda_oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, dp, dp,
                                       ctypes.c_int, dp, dp, dp, dp, dp, dp]
        lib.kda_oracle_bwd.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _f64(x) -> np.ndarray:
    """Exact widening of a torch tensor or array to a contiguous fp64 array."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any device, any float dtype)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads_available() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def kda_fwd_packed(q, k, v, g, beta, h0=None, cu_seqlens=None, nthreads: int = 0):
    """Oracle on packed sequences.

    q, k, g: [T_total, H, d_k]; v: [T_total, H, d_v]; beta: [T_total, H];
    h0: [N, H, d_k, d_v] or None; cu_seqlens: [N+1] token offsets (None: one
    sequence).  Returns (o [T_total, H, d_v], hT [N, H, d_k, d_v], threads).
    """
    q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
    T, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (T, H, dk) and g.shape == (T, H, dk)
    assert v.shape == (T, H, dv) and beta.shape == (T, H)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    assert cu[-1] == T
    if h0 is not None:
        assert h0.shape == (N, H, dk, dv)
    o = np.zeros((T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    used = _lib().kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                 N, H, dk, dv, int(nthreads), _ptr(o), _ptr(hT))
    if used < 0:
        raise ValueError("kda_oracle_fwd rejected its arguments")
    return o, hT, used


def kda_fwd(q, k, v, g, beta, h0=None, cu_seqlens=None, nthreads: int = 0):
    """Oracle on [B, T, H, d] inputs (B equal-length sequences) or, with
    cu_seqlens, on packed inputs of shape [1, T_total, H, d].

    Returns (o [B, T, H, d_v] fp64, hT [N, H, d_k, d_v] fp64) where N = B
    without cu_seqlens and N = len(cu_seqlens) - 1 with it.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        assert B == 1, "packed inputs have B == 1"
        cu = cu_seqlens
    o, hT, _ = kda_fwd_packed(q.reshape(B * T, H, dk), k.reshape(B * T, H, dk),
                              v.reshape(B * T, H, dv), g.reshape(B * T, H, dk),
                              beta.reshape(B * T, H), h0, cu, nthreads)
    return o.reshape(B, T, H, dv), hT


def kda_decode_step(q, k, v, g, beta, S, nthreads: int = 0):
    """One decode token per sequence: q, k, g [N, H, d_k]; v [N, H, d_v];
    beta [N, H]; S [N, H, d_k, d_v].  Returns (o [N, H, d_v], S_new)."""
    q, k, v, g, beta, S = map(_f64, (q, k, v, g, beta, S))
    N = q.shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    o, hT, _ = kda_fwd_packed(q, k, v, g, beta, S, cu, nthreads)
    return o, hT


def kda_decode_verify(q, k, v, g, beta, S, nthreads: int = 0):
    """K drafted tokens per sequence, run from the state S (which is not changed):
    q, k, g [N, K, H, d_k]; v [N, K, H, d_v]; beta [N, K, H]; S [N, H, d_k, d_v].
    Returns o [N, K, H, d_v]: o[n, t] is the read of the state after drafted tokens
    0..t of sequence n, i.e. the recurrence over the K tokens from S."""
    q, k, v, g, beta, S = map(_f64, (q, k, v, g, beta, S))
    N, K, H, dk = q.shape
    dv = v.shape[3]
    cu = np.arange(N + 1, dtype=np.int64) * K
    o, _, _ = kda_fwd_packed(q.reshape(N * K, H, dk), k.reshape(N * K, H, dk),
                             v.reshape(N * K, H, dv), g.reshape(N * K, H, dk),
                             beta.reshape(N * K, H), S, cu, nthreads)
    return o.reshape(N, K, H, dv)


def kda_decode_commit(k, v, g, beta, accepted, S, nthreads: int = 0):
    """The state of every sequence after only its first accepted[n] drafted tokens
    (k, g [N, K, H, d_k]; v [N, K, H, d_v]; beta [N, K, H]; S [N, H, d_k, d_v];
    accepted [N] integers in [0, K]): the recurrence from S over that prefix, the
    rejected tokens never entering the state.  Returns the new states [N, H, d_k, d_v]."""
    k, v, g, beta, S = map(_f64, (k, v, g, beta, S))
    if hasattr(accepted, "detach"):
        accepted = accepted.detach().cpu().numpy()
    acc = np.asarray(accepted, dtype=np.int64)
    N, K, H, dk = k.shape
    dv = v.shape[3]
    if acc.shape != (N,) or (acc < 0).any() or (acc > K).any():
        raise ValueError("accepted must hold N counts in [0, K]")
    take = lambda x: np.ascontiguousarray(  # noqa: E731
        np.concatenate([x[n, :acc[n]] for n in range(N)], axis=0))
    cu = np.concatenate([[0], np.cumsum(acc)]).astype(np.int64)
    kp, vp, gp, bp = take(k), take(v), take(g), take(beta)
    qp = np.zeros_like(kp)                     # outputs are not needed here
    _, hT, _ = kda_fwd_packed(qp, kp, vp, gp, bp, S, cu, nthreads)
    return hT


def kda_bwd_packed(q, k, v, g, beta, h0, cu_seqlens, do, dhT=None, nthreads: int = 0):
    """Gradient of the recurrence on packed sequences (layouts as kda_fwd_packed):
    given do = dL/do [T_total, H, d_v] and dhT = dL/dhT [N, H, d_k, d_v] (None: zero),
    returns (dq, dk, dv, dg, dbeta, dh0) = dL/d(input) in fp64."""
    q, k, v, g, beta, h0, do, dhT = map(_f64, (q, k, v, g, beta, h0, do, dhT))
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    assert cu[-1] == T and do.shape == (T, H, dv)
    if dhT is not None:
        assert dhT.shape == (N, H, dk, dv)
    dq, dkk, dg = (np.zeros((T, H, dk)) for _ in range(3))
    dvv = np.zeros((T, H, dv))
    db = np.zeros((T, H))
    dh0 = np.zeros((N, H, dk, dv))
    used = _lib().kda_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, H, dk, dv,
                                 _ptr(do), _ptr(dhT), int(nthreads), _ptr(dq), _ptr(dkk),
                                 _ptr(dvv), _ptr(dg), _ptr(db), _ptr(dh0))
    if used < 0:
        raise ValueError("kda_oracle_bwd rejected its arguments")
    return dq, dkk, dvv, dg, db, dh0


def kda_bwd(q, k, v, g, beta, h0, do, dhT=None, cu_seqlens=None, nthreads: int = 0):
    """Gradient on [B, T, H, d] inputs (or packed [1, T_total, H, d] with cu_seqlens):
    returns (dq, dk, dv, dg, dbeta, dh0) shaped like the inputs (dh0 [N, H, d_k, d_v])."""
    q, k, v, g, beta, do = map(_f64, (q, k, v, g, beta, do))
    B, T, H, dk = q.shape
    dv = v.shape[3]
    cu = np.arange(B + 1, dtype=np.int64) * T if cu_seqlens is None else cu_seqlens
    r = kda_bwd_packed(q.reshape(B * T, H, dk), k.reshape(B * T, H, dk), v.reshape(B * T, H, dv),
                       g.reshape(B * T, H, dk), beta.reshape(B * T, H), h0, cu,
                       do.reshape(B * T, H, dv), dhT, nthreads)
    dq, dkk, dvv, dg, db, dh0 = r
    return (dq.reshape(B, T, H, dk), dkk.reshape(B, T, H, dk), dvv.reshape(B, T, H, dv),
            dg.reshape(B, T, H, dk), db.reshape(B, T, H), dh0)
