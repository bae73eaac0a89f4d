"""Pins of the fp64 oracle against facts other than itself (CPU only).

Every test compares the oracle's token loop with a route that does not share
its arithmetic: dense operator products, exact rational arithmetic, the
chunkwise algebra, and closed forms of special cases.  The recurrence is the
single-head KDA update of the "Kimi K3" open-weights field notes
(ailearn.mscapital.top/kimi-k3.html), panel "KDA 单头递归":
decay per key channel, then delta-rule erase and write, then the query reads
the updated state.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.oracle_helpers import as_batch, brute_force, chunked, exact_rational, rand_chain


def run_chain(q, k, v, g, beta, S0):
    o, hT = oracle.kda_fwd(*as_batch(q, k, v, g, beta), h0=S0[None, None])
    return o[0, :, 0, :], hT[0, 0]


@pytest.mark.parametrize("T,dk,dv,seed", [(1, 3, 2, 0), (5, 4, 3, 1), (12, 4, 4, 2), (9, 2, 5, 3)])
def test_brute_force_operator_products(T, dk, dv, seed):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = rand_chain(rng, T, dk, dv, unit_keys=False)
    o_ref, S_ref = brute_force(q, k, v, g, beta, S0)
    o, S = run_chain(q, k, v, g, beta, S0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)


def test_exact_rational_arithmetic():
    """T=4, d_k=2, d_v=3 in exact rationals.  alpha = exp(g) is a power of two,
    so exp(log(alpha)) reaches the oracle within an ulp; k, q, v, beta are dyadic
    and exact in fp64."""
    rng = np.random.default_rng(11)
    T, dk, dv = 4, 2, 3
    dy = lambda x: Fraction(int(round(x * 64)), 64)  # noqa: E731
    k = [[dy(x) for x in rng.uniform(-1, 1, dk)] for _ in range(T)]
    q = [[dy(x) for x in rng.uniform(-1, 1, dk)] for _ in range(T)]
    v = [[dy(x) for x in rng.uniform(-2, 2, dv)] for _ in range(T)]
    beta = [dy(x) for x in rng.uniform(0, 1, T)]
    alpha = [[Fraction(1, 2 ** int(e)) for e in rng.integers(0, 4, dk)] for _ in range(T)]
    S0 = [[dy(x) for x in rng.uniform(-1, 1, dv)] for _ in range(dk)]
    outs, S = exact_rational(q, k, v, alpha, beta, S0)
    f = lambda a: np.array(a, dtype=np.float64)  # noqa: E731
    g = np.log(f(alpha))
    np.testing.assert_allclose(np.exp(g), f(alpha), rtol=4e-16, atol=0)
    o, hT = run_chain(f(q), f(k), f(v), g, f(beta), f(S0))
    np.testing.assert_allclose(o, f(outs), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(hT, f(S), rtol=1e-14, atol=1e-14)


def test_beta_zero_is_pure_decay():
    """beta = 0: S_T = Diag(exp(sum_t g_t)) S_0 and o_t = (Diag(exp G_t) S_0)^T q_t."""
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = rand_chain(rng, 20, 6, 5)
    beta[:] = 0.0
    o, S = run_chain(q, k, v, g, beta, S0)
    G = np.cumsum(g, axis=0)
    np.testing.assert_allclose(S, np.exp(G[-1])[:, None] * S0, rtol=1e-13, atol=0)
    o_ref = np.stack([(np.exp(G[t])[:, None] * S0).T @ q[t] for t in range(20)])
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-15)


def test_unit_write_retrieves_last_value():
    """beta_t = 1, |k_t| = 1, q_t = k_t: the delta rule overwrites the value
    stored under k_t, so o_t = v_t for every t, whatever the decay and the
    prior state."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta, S0 = rand_chain(rng, 30, 8, 5)
    beta[:] = 1.0
    S0 = 3.0 * rng.standard_normal(S0.shape)
    o, _ = run_chain(k.copy(), k, v, g, beta, S0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


def test_orthonormal_keys_are_an_associative_memory():
    """alpha = 1, beta = 1, orthonormal keys and S_0 = 0: afterwards S^T k_j = v_j
    for every stored j, and S = K^T V exactly."""
    rng = np.random.default_rng(7)
    dk, dv, T = 8, 4, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T.copy()
    v = rng.standard_normal((T, dv))
    g = np.zeros((T, dk))
    beta = np.ones(T)
    o, S = run_chain(k.copy(), k, v, g, beta, np.zeros((dk, dv)))
    np.testing.assert_allclose(S, k.T @ v, atol=1e-14)
    np.testing.assert_allclose(S.T @ k.T, v.T, atol=1e-14)


def test_scalar_key_dimension_closed_form():
    """d_k = 1: s_t = a_t s_{t-1} + b_t k_t v_t with a_t = (1 - b_t k_t^2) exp(g_t),
    whose closed form is s_T = (prod a) s_0 + sum_t (prod_{u>t} a_u) b_t k_t v_t."""
    rng = np.random.default_rng(8)
    T, dv = 25, 3
    k = rng.uniform(-1.2, 1.2, (T, 1))
    q = rng.standard_normal((T, 1))
    v = rng.standard_normal((T, dv))
    g = -rng.uniform(0, 2, (T, 1))
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((1, dv))
    a = (1.0 - beta * k[:, 0] ** 2) * np.exp(g[:, 0])
    tail = np.array([np.prod(a[t + 1:]) for t in range(T)])
    sT = np.prod(a) * S0[0] + ((tail * beta * k[:, 0])[:, None] * v).sum(0)
    o, S = run_chain(q, k, v, g, beta, S0)
    np.testing.assert_allclose(S[0], sT, rtol=1e-12, atol=1e-13)
    # o_T = q_T s_T
    np.testing.assert_allclose(o[-1], q[-1, 0] * sT, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("C", [1, 2, 16, 64, 100])
def test_chunked_evaluation_equals_recurrence(C):
    rng = np.random.default_rng(9)
    T, dk, dv = 100, 8, 6
    q, k, v, g, beta, S0 = rand_chain(rng, T, dk, dv, gmin=-1.0)
    o_ref, S_ref = run_chain(q, k, v, g, beta, S0)
    o, S = chunked(q, k, v, g, beta, S0, C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S, S_ref, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("C", [16, 64])
def test_chunked_at_the_decay_bound(C):
    """g close to -5 (the stated lower bound) inside 64-token chunks."""
    rng = np.random.default_rng(10)
    T, dk, dv = 128, 8, 4
    q, k, v, g, beta, S0 = rand_chain(rng, T, dk, dv)
    g = -5.0 * (1.0 - 1e-3 * rng.random((T, dk)))
    o_ref, S_ref = run_chain(q, k, v, g, beta, S0)
    o, S = chunked(q, k, v, g, beta, S0, C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-9, atol=1e-12)


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(12)
    q, k, v1, g, beta, S1 = rand_chain(rng, 15, 5, 4)
    v2 = rng.standard_normal(v1.shape)
    S2 = rng.standard_normal(S1.shape)
    a, b = 0.7, -1.9
    o1, T1 = run_chain(q, k, v1, g, beta, S1)
    o2, T2 = run_chain(q, k, v2, g, beta, S2)
    o3, T3 = run_chain(q, k, a * v1 + b * v2, g, beta, a * S1 + b * S2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, atol=1e-12)
    np.testing.assert_allclose(T3, a * T1 + b * T2, atol=1e-12)


def test_value_columns_are_independent():
    rng = np.random.default_rng(13)
    q, k, v, g, beta, S0 = rand_chain(rng, 15, 5, 6)
    perm = rng.permutation(6)
    o, S = run_chain(q, k, v, g, beta, S0)
    op, Sp = run_chain(q, k, v[:, perm], g, beta, S0[:, perm])
    np.testing.assert_allclose(op, o[:, perm], atol=1e-14)
    np.testing.assert_allclose(Sp, S[:, perm], atol=1e-14)


def test_split_run_resumes_from_final_state():
    rng = np.random.default_rng(14)
    q, k, v, g, beta, S0 = rand_chain(rng, 40, 6, 5)
    o, S = run_chain(q, k, v, g, beta, S0)
    o1, S1 = run_chain(q[:17], k[:17], v[:17], g[:17], beta[:17], S0)
    o2, S2 = run_chain(q[17:], k[17:], v[17:], g[17:], beta[17:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, atol=1e-14)
    np.testing.assert_allclose(S2, S, atol=1e-14)


def test_varlen_equals_independent_runs():
    rng = np.random.default_rng(15)
    H, dk, dv = 3, 4, 5
    lengths = [7, 0, 1, 12]
    Tt = sum(lengths)
    q = rng.standard_normal((1, Tt, H, dk))
    k = rng.standard_normal((1, Tt, H, dk)) * 0.5
    v = rng.standard_normal((1, Tt, H, dv))
    g = -rng.uniform(0, 5, (1, Tt, H, dk))
    beta = rng.uniform(0, 1, (1, Tt, H))
    h0 = rng.standard_normal((len(lengths), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, hT = oracle.kda_fwd(q, k, v, g, beta, h0=h0, cu_seqlens=cu)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        on, hn = oracle.kda_fwd(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b],
                                h0=h0[n:n + 1])
        np.testing.assert_array_equal(o[:, a:b], on)
        np.testing.assert_array_equal(hT[n], hn[0])
    # an empty sequence returns its initial state untouched
    np.testing.assert_array_equal(hT[1], h0[1])


def test_heads_are_independent_and_batched():
    rng = np.random.default_rng(16)
    B, T, H, dk, dv = 2, 9, 3, 4, 4
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) * 0.5
    v = rng.standard_normal((B, T, H, dv))
    g = -rng.uniform(0, 5, (B, T, H, dk))
    beta = rng.uniform(0, 1, (B, T, H))
    h0 = rng.standard_normal((B, H, dk, dv))
    o, hT = oracle.kda_fwd(q, k, v, g, beta, h0=h0)
    for b in range(B):
        for h in range(H):
            oc, Sc = run_chain(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h], beta[b, :, h], h0[b, h])
            np.testing.assert_array_equal(o[b, :, h], oc)
            np.testing.assert_array_equal(hT[b, h], Sc)


def test_chained_decode_equals_prefill():
    rng = np.random.default_rng(17)
    N, H, dk, dv, steps = 2, 2, 4, 3, 6
    q = rng.standard_normal((steps, N, H, dk))
    k = rng.standard_normal((steps, N, H, dk)) * 0.5
    v = rng.standard_normal((steps, N, H, dv))
    g = -rng.uniform(0, 5, (steps, N, H, dk))
    beta = rng.uniform(0, 1, (steps, N, H))
    S = rng.standard_normal((N, H, dk, dv))
    S_dec = S.copy()
    outs = []
    for s in range(steps):
        o, S_dec = oracle.kda_decode_step(q[s], k[s], v[s], g[s], beta[s], S_dec)
        outs.append(o)
    tr = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1))  # [steps, N, ...] -> [N, steps, ...]  # noqa: E731
    o_pf, S_pf = oracle.kda_fwd(tr(q), tr(k), tr(v), tr(g), tr(beta), h0=S)
    np.testing.assert_allclose(np.stack(outs, 1), o_pf, atol=1e-14)
    np.testing.assert_allclose(S_dec, S_pf, atol=1e-14)


def test_state_norm_growth_bound():
    """With g <= 0 and 0 <= beta |k|^2 <= 2 the transition is non-expansive, so
    ||S_t||_F <= ||S_{t-1}||_F + beta_t |k_t| |v_t|."""
    rng = np.random.default_rng(18)
    q, k, v, g, beta, S0 = rand_chain(rng, 50, 6, 4)
    S = S0
    for t in range(50):
        _, Sn = run_chain(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], S)
        bound = np.linalg.norm(S) + beta[t] * np.linalg.norm(k[t]) * np.linalg.norm(v[t])
        assert np.linalg.norm(Sn) <= bound * (1 + 1e-12)
        S = Sn


def test_windowed_restart_bound():
    """The influence of S_{t0} on S_t is bounded by exp(sum_{u in (t0, t]} max_c g_uc)
    (each transition has norm <= max_c exp(g_uc)), which justifies checking long
    runs on windows: a run started at zero L tokens early differs from the full run
    by at most that factor times ||S_{t0}||."""
    rng = np.random.default_rng(19)
    T, dk, dv, L = 300, 8, 4, 120
    q, k, v, g, beta, S0 = rand_chain(rng, T, dk, dv)
    o, S = run_chain(q, k, v, g, beta, S0)
    _, Smid = run_chain(q[:T - L], k[:T - L], v[:T - L], g[:T - L], beta[:T - L], S0)
    o_w, S_w = run_chain(q[T - L:], k[T - L:], v[T - L:], g[T - L:], beta[T - L:], np.zeros_like(S0))
    factor = math.exp(g[T - L:].max(axis=1).sum())
    assert np.linalg.norm(S - S_w, 2) <= factor * np.linalg.norm(Smid, 2) * (1 + 1e-9) + 1e-14


def test_oracle_rejects_bad_offsets():
    z = np.zeros((1, 4, 1, 2))
    with pytest.raises(ValueError):
        oracle.kda_fwd(z, z, z, z, np.zeros((1, 4, 1)), cu_seqlens=np.array([0, 3, 2, 4]))


def _draft_batch(rng, N, K, H, dk, dv):
    """N sequences x H heads of K drafted tokens, [N, K, H, d] layouts, plus states."""
    chains = [[rand_chain(rng, K, dk, dv) for _ in range(H)] for _ in range(N)]
    st = lambda i: np.stack([np.stack([chains[n][h][i] for h in range(H)], axis=1)  # noqa: E731
                             for n in range(N)])
    q, k, v, g = st(0), st(1), st(2), st(3)
    beta = np.stack([np.stack([chains[n][h][4] for h in range(H)], axis=1) for n in range(N)])
    S = np.stack([np.stack([chains[n][h][5] for h in range(H)]) for n in range(N)])
    return chains, q, k, v, g, beta, S


def test_decode_verify_equals_brute_force_on_every_prefix():
    """Verify = the recurrence over the K drafted tokens from S, read after each token:
    against the dense operator products, chain by chain; S itself is not changed."""
    rng = np.random.default_rng(40)
    N, K, H, dk, dv = 3, 5, 2, 4, 3
    chains, q, k, v, g, beta, S = _draft_batch(rng, N, K, H, dk, dv)
    S_before = S.copy()
    o = oracle.kda_decode_verify(q, k, v, g, beta, S)
    assert o.shape == (N, K, H, dv) and np.array_equal(S, S_before)
    for n in range(N):
        for h in range(H):
            cq, ck, cv, cg, cb, _ = chains[n][h]
            o_bf, _ = brute_force(cq, ck, cv, cg, cb, S[n, h])
            assert np.allclose(o[n, :, h], o_bf, rtol=1e-12, atol=1e-12)


def test_decode_commit_keeps_only_the_accepted_prefix():
    """Commit = the state after only the first a_n drafted tokens (a different a_n per
    sequence, 0 and K included): against the dense operator products on that prefix;
    a_n = 0 returns the state exactly; counts outside [0, K] are refused."""
    rng = np.random.default_rng(41)
    N, K, H, dk, dv = 4, 6, 2, 5, 3
    chains, q, k, v, g, beta, S = _draft_batch(rng, N, K, H, dk, dv)
    acc = np.array([0, 3, 6, 1])
    S_new = oracle.kda_decode_commit(k, v, g, beta, acc, S)
    for n in range(N):
        for h in range(H):
            if acc[n] == 0:
                assert np.array_equal(S_new[n, h], S[n, h])
                continue
            cq, ck, cv, cg, cb, _ = chains[n][h]
            a = acc[n]
            _, S_bf = brute_force(cq[:a], ck[:a], cv[:a], cg[:a], cb[:a], S[n, h])
            assert np.allclose(S_new[n, h], S_bf, rtol=1e-12, atol=1e-12)
    # a rejected token changes nothing: the tail of the draft is irrelevant
    k2, v2, g2 = k.copy(), v.copy(), g.copy()
    k2[1, 3:] = rng.standard_normal(k2[1, 3:].shape)
    v2[1, 3:] += 1.0
    g2[1, 3:] = -4.0
    assert np.array_equal(oracle.kda_decode_commit(k2, v2, g2, beta, acc, S)[1], S_new[1])
    with pytest.raises(ValueError):
        oracle.kda_decode_commit(k, v, g, beta, np.array([0, 7, 1, 1]), S)
    with pytest.raises(ValueError):
        oracle.kda_decode_commit(k, v, g, beta, np.array([0, -1, 1, 1]), S)
