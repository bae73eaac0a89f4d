"""Independent evaluations of the KDA recurrence used to pin the oracle.

Each helper reaches the recurrence's result by a route other than the oracle's
token loop (dense operator products, exact rational arithmetic, the chunkwise
algebra, closed forms), so a mistake in the oracle shows up as a mismatch.

Recurrence (single head): S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1}
+ b_t k_t v_t^T and o_t = S_t^T q_t, from the "Kimi K3" open-weights field
notes (ailearn.mscapital.top/kimi-k3.html), panel "KDA 单头递归".
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def rand_chain(rng, T, dk, dv, unit_keys=True, gmin=-5.0):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        q /= np.linalg.norm(q, axis=1, keepdims=True) * np.sqrt(dk)
    v = rng.standard_normal((T, dv))
    g = gmin / (1.0 + np.exp(-(rng.standard_normal((T, dk)) - 1.0)))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    return q, k, v, g, beta, S0


def transition(k, g, beta):
    """Dense transition operator M_t = (I - b k k^T) Diag(exp g), d_k x d_k."""
    dk = k.shape[0]
    return (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(np.exp(g))


def brute_force(q, k, v, g, beta, S0):
    """S_t = M_t ... M_1 S0 + sum_{i<=t} M_t ... M_{i+1} b_i k_i v_i^T, each S_t
    formed from scratch by dense products (O(T^2) operator products)."""
    T, dk = k.shape
    Ms = [transition(k[t], g[t], beta[t]) for t in range(T)]
    outs, S = [], None
    for t in range(T):
        P = np.eye(dk)
        S = np.zeros_like(S0)
        for i in range(t, -1, -1):          # i = t, t-1, ..., 0
            S = S + P @ (beta[i] * np.outer(k[i], v[i]))
            P = P @ Ms[i]
        S = S + P @ S0
        outs.append(S.T @ q[t])
    return np.array(outs), S


def exact_rational(q, k, v, alpha, beta, S0):
    """The recurrence in exact rational arithmetic (Fractions).  alpha is the
    decay factor exp(g) itself, given as Fractions."""
    T, dk = len(k), len(k[0])
    dv = len(v[0])
    S = [[Fraction(S0[i][j]) for j in range(dv)] for i in range(dk)]
    outs = []
    for t in range(T):
        D = [[alpha[t][i] * S[i][j] for j in range(dv)] for i in range(dk)]
        # (I - b k k^T) D + b k v^T as explicit matrix arithmetic
        E = [[(1 if i == m else 0) - beta[t] * k[t][i] * k[t][m] for m in range(dk)]
             for i in range(dk)]
        S = [[sum(E[i][m] * D[m][j] for m in range(dk)) + beta[t] * k[t][i] * v[t][j]
              for j in range(dv)] for i in range(dk)]
        outs.append([sum(S[i][j] * q[t][i] for i in range(dk)) for j in range(dv)])
    return outs, S


def chunked(q, k, v, g, beta, S0, C):
    """Chunkwise (UT / WY) evaluation with chunk length C, derived from the
    recurrence: within a chunk with inclusive cumulative log-decay G_r,

      A_ri  = b_r sum_c k_rc k_ic exp(G_rc - G_ic)          (i < r)
      T     = (I + A)^{-1}
      W     = T Diag(b) (K * exp(G)),  U = T Diag(b) V
      Delta = U - W S                                       (the delta-rule errors)
      O     = (Q * exp(G)) S + [i <= r] (sum_c q_rc k_ic exp(G_rc - G_ic)) Delta
      S    <- Diag(exp(G_C)) S + (K * exp(G_C - G))^T Delta
    """
    T, dk = k.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, b = q[sl], k[sl], v[sl], beta[sl]
        L = K.shape[0]
        G = np.cumsum(g[sl], axis=0)
        lower = np.tril(np.ones((L, L), dtype=bool))
        with np.errstate(over="ignore", invalid="ignore"):
            D = np.exp(G[:, None, :] - G[None, :, :])
            Akk = np.einsum("rc,ic,ric->ri", K, K, D)
            Aqk = np.einsum("rc,ic,ric->ri", Q, K, D)
        Akk = np.where(np.tril(lower, -1), Akk, 0.0) * b[:, None]
        Aqk = np.where(lower, Aqk, 0.0)
        Tm = np.linalg.inv(np.eye(L) + Akk)
        gam = np.exp(G)
        W = Tm @ (b[:, None] * K * gam)
        U = Tm @ (b[:, None] * V)
        Delta = U - W @ S
        o[sl] = (Q * gam) @ S + Aqk @ Delta
        Kt = K * np.exp(G[-1][None, :] - G)
        S = gam[-1][:, None] * S + Kt.T @ Delta
    return o, S


def as_batch(q, k, v, g, beta):
    """[T, d] single-chain arrays -> [1, T, 1, d] oracle inputs."""
    return (q[None, :, None, :], k[None, :, None, :], v[None, :, None, :],
            g[None, :, None, :], beta[None, :, None])
