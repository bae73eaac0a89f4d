"""Pins of the oracle's gradient (CPU only).

The gradient ``oracle.kda_bwd`` is reverse accumulation through the recurrence of the
"Kimi K3" field notes, panel "KDA 单头递归".  It is pinned to something other than
itself: central finite differences of the (separately pinned) forward oracle,
element by element on tiny chains and along random directions on packed batches
that span several of its recompute segments, with empty sequences and nonzero
initial and final-state gradients.  Planted mistakes in its C source must fail
those pins.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle
import oracle.build as obuild
import oracle.kda_oracle as ko


def _batch(rng, lengths, H, dk, dv, gmin=-2.0):
    T = int(sum(lengths))
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    g = gmin / (1.0 + np.exp(-rng.standard_normal((T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    N = len(lengths)
    h0 = 0.3 * rng.standard_normal((N, H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    do = rng.standard_normal((T, H, dv))
    dhT = rng.standard_normal((N, H, dk, dv))
    return [q, k, v, g, beta, h0], cu, do, dhT


def _loss(args, cu, do, dhT):
    o, hT, _ = oracle.kda_fwd_packed(*args, cu)
    return float((o * do).sum() + (hT * dhT).sum())


NAMES = ["q", "k", "v", "g", "beta", "h0"]


def test_gradient_matches_finite_differences_elementwise():
    rng = np.random.default_rng(3)
    args, cu, do, dhT = _batch(rng, [4, 0, 5], H=2, dk=3, dv=4)
    grads = oracle.kda_bwd_packed(*args, cu, do, dhT)
    eps = 1e-6
    for ai, (a, gr) in enumerate(zip(args, grads)):
        assert gr.shape == a.shape
        for idx in np.ndindex(a.shape):
            ap = [x.copy() for x in args]
            am = [x.copy() for x in args]
            ap[ai][idx] += eps
            am[ai][idx] -= eps
            fd = (_loss(ap, cu, do, dhT) - _loss(am, cu, do, dhT)) / (2 * eps)
            assert abs(fd - gr[idx]) <= 1e-6 * (1.0 + abs(fd)), (NAMES[ai], idx, fd, gr[idx])


@pytest.mark.parametrize("lengths", [[150], [70, 0, 130, 1]])
def test_gradient_matches_finite_differences_along_directions(lengths):
    """Longer chains (across the oracle's 64-token recompute segments): the derivative
    of the loss along a random direction in each input equals the gradient's inner
    product with it."""
    rng = np.random.default_rng(len(lengths))
    args, cu, do, dhT = _batch(rng, lengths, H=2, dk=8, dv=6)
    grads = oracle.kda_bwd_packed(*args, cu, do, dhT)
    eps = 1e-6
    for ai, (a, gr) in enumerate(zip(args, grads)):
        d = rng.standard_normal(a.shape)
        ap = [x.copy() for x in args]
        am = [x.copy() for x in args]
        ap[ai] += eps * d
        am[ai] -= eps * d
        fd = (_loss(ap, cu, do, dhT) - _loss(am, cu, do, dhT)) / (2 * eps)
        an = float((gr * d).sum())
        assert abs(fd - an) <= 1e-6 * (1.0 + abs(fd)), (NAMES[ai], fd, an)


def test_gradient_of_an_empty_sequence_passes_through():
    """An empty sequence's final state is its initial state: dh0 = dhT and nothing else."""
    rng = np.random.default_rng(9)
    args, cu, do, dhT = _batch(rng, [0, 3], H=1, dk=2, dv=2)
    grads = oracle.kda_bwd_packed(*args, cu, do, dhT)
    assert np.array_equal(grads[5][0], dhT[0])


def test_batched_wrapper_matches_packed():
    rng = np.random.default_rng(4)
    args, cu, do, dhT = _batch(rng, [7, 7], H=2, dk=3, dv=3)
    q, k, v, g, beta, h0 = args
    sh = lambda x: x.reshape(2, 7, *x.shape[1:])  # noqa: E731
    r1 = oracle.kda_bwd(sh(q), sh(k), sh(v), sh(g), sh(beta), h0, sh(do), dhT)
    r2 = oracle.kda_bwd_packed(*args, cu, do, dhT)
    for a, b in zip(r1, r2):
        assert np.array_equal(a.reshape(b.shape), b)


# ---- planted mistakes in the gradient's C source must fail the pins ----
BWD_MUTANTS = {
    "read_gradient_dropped": ("G[i * dv + j] += qt[i] * dot[j];", "G[i * dv + j] += 0.0;"),
    "dq_from_old_state": ("x += St[i * dv + j] * dot[j];", "x += Sprev[i * dv + j] * dot[j];"),
    "erase_term_of_dk_dropped": ("dkt[i] = bt * w[i] - x;", "dkt[i] = bt * w[i];"),
    "dv_without_beta": ("dd[j] *= bt;", "dd[j] *= 1.0;"),
    "decay_not_applied_backward": ("G[i * dv + j] = a_i * gp;", "G[i * dv + j] = gp;"),
    "dg_against_old_state": ("x += Sp[i * dv + j] * gp;", "x += Sprev[i * dv + j] * gp;"),
    "erase_not_in_state_gradient": ("const double gp = G[i * dv + j] - kt[i] * dd[j];",
                                    "const double gp = G[i * dv + j];"),
}


def _load_bwd(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_int64)
    lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int, dp, dp]
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int64, dp, dp, ctypes.c_int, dp, dp,
                                   dp, dp, dp, dp]
    lib.kda_oracle_bwd.restype = ctypes.c_int
    return lib


def _pins_pass():
    try:
        test_gradient_matches_finite_differences_elementwise()
        test_gradient_matches_finite_differences_along_directions([70, 0, 130, 1])
        return True
    except AssertionError:
        return False


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_planted_gradient_mistake_fails_a_pin(name, tmp_path, monkeypatch):
    src = open(obuild.SRC).read()
    old, new = BWD_MUTANTS[name]
    assert src.count(old) == 1, name
    # only the gradient is mutated: the forward the finite differences use stays intact
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    out = str(tmp_path / "libmut.so")
    obuild.build(force=True, src=str(path), out=out)
    monkeypatch.setattr(ko, "_LIB", _load_bwd(out))
    assert not _pins_pass(), f"mutant {name} passed every gradient pin"


def test_unmutated_gradient_passes_the_pins():
    assert _pins_pass()
    assert os.path.exists(obuild.LIB)
