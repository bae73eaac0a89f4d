"""The chunk algebra the tensor-core path is built on, in fp64, against the oracle.

The prefill kernels never run the recurrence token by token.  The intra-chunk
kernel turns every 64-token chunk into an affine map on the state,

    S_out = Diag(exp G_C) S_in + M' S_in + R,      O = Q' S_in + O0,

with M' = -Kt^T W, R = Kt^T U, Q' = Qg - Aqk W, O0 = Aqk U, [W | U] = T' [K exp G | V]
and T' = (I + A)^-1 Diag(beta), and the state pass applies the maps in order.  This
test writes that decomposition out in fp64 (no rounding to bf16: it checks the
algebra, not the kernels' precision) and compares it with the token-by-token oracle,
and checks the range claim behind the 16-token sub-tile references: with
g in (-5, 0], every decay factor the kernels form stays within e^40 and every
pairwise factor between sub-tiles is at most 1.
"""
import numpy as np
import pytest

import oracle

C, ST = 64, 16      # chunk and sub-tile lengths of the tensor-core path
REF = ST // 2 - 1   # reference row inside each sub-tile (its 8th row)


def chunk_map(q, k, v, g, beta):
    """Affine record of one chunk (L <= C rows; d_k columns of q, k, g; d_v of v)."""
    L = q.shape[0]
    G = np.cumsum(g, axis=0)                               # inclusive in-chunk cumsum
    GC = G[-1]
    # pairwise decays through the sub-tile references: r in sub-tile a, i in sub-tile b
    ref = np.array([min(ST * (r // ST) + REF, L - 1) for r in range(L)])
    E = np.empty((L, L, q.shape[1]))
    for r in range(L):
        for i in range(L):
            E[r, i] = np.exp(G[r] - G[ref[r]]) * np.exp(G[ref[r]] - G[ref[i]]) * \
                np.exp(G[ref[i]] - G[i])
    A = np.zeros((L, L))
    Aqk = np.zeros((L, L))
    for r in range(L):
        for i in range(L):
            if i < r:
                A[r, i] = beta[r] * np.sum(k[r] * k[i] * E[r, i])
            if i <= r:
                Aqk[r, i] = np.sum(q[r] * k[i] * E[r, i])
    Tp = np.linalg.solve(np.eye(L) + A, np.diag(beta))    # T' = (I + A)^-1 Diag(beta)
    W = Tp @ (k * np.exp(G))
    U = Tp @ v
    Kt = k * np.exp(GC - G)
    return dict(M=-(Kt.T @ W), R=Kt.T @ U, Qp=q * np.exp(G) - Aqk @ W, O0=Aqk @ U,
                gC=np.exp(GC), E=E, G=G, ref=ref)


def run_maps(q, k, v, g, beta, S):
    outs = []
    for t0 in range(0, q.shape[0], C):
        sl = slice(t0, t0 + C)
        m = chunk_map(q[sl], k[sl], v[sl], g[sl], beta[sl])
        outs.append(m["Qp"] @ S + m["O0"])
        S = m["gC"][:, None] * S + m["M"] @ S + m["R"]
    return np.vstack(outs), S


def inputs(T, dk, dv, seed, g_fill=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * np.sqrt(dk)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -5.0 / (1.0 + np.exp(-(rng.standard_normal((T, dk)) - 3.0)))
    if g_fill is not None:
        g = np.full((T, dk), g_fill)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = 0.1 * rng.standard_normal((dk, dv))
    return q, k, v, g, beta, S0


def reference(q, k, v, g, beta, S0):
    o, hT = oracle.kda_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                           g[None, :, None], beta[None, :, None], S0[None, None])
    return o[0, :, 0], hT[0, 0]


@pytest.mark.parametrize("T", [64, 150, 256])
def test_affine_chunk_maps_equal_the_recurrence(T):
    """Full chunks and a ragged last chunk (150 = 2 x 64 + 22)."""
    q, k, v, g, beta, S0 = inputs(T, 12, 10, seed=T)
    o, S = run_maps(q, k, v, g, beta, S0)
    o_ref, S_ref = reference(q, k, v, g, beta, S0)
    assert np.abs(o - o_ref).max() <= 1e-11 * max(1.0, np.abs(o_ref).max())
    assert np.abs(S - S_ref).max() <= 1e-11 * max(1.0, np.abs(S_ref).max())


def test_segment_maps_compose():
    """The time split's premise: a segment of chunks acts on the state as one affine
    map S -> P S + R, with R the state it reaches from zero and P the state it
    reaches from the identity with the values zeroed (the two halves of the widened
    state the map pass runs), and segment maps compose in order."""
    T, dk, dv = 200, 6, 5
    q, k, v, g, beta, S0 = inputs(T, dk, dv, seed=7)

    def seg_map(t0, t1):
        sl = slice(t0, t1)
        _, R = run_maps(q[sl], k[sl], v[sl], g[sl], beta[sl], np.zeros((dk, dv)))
        _, P = run_maps(q[sl], k[sl], np.zeros((t1 - t0, dk)), g[sl], beta[sl], np.eye(dk))
        return P, R

    P1, R1 = seg_map(0, 128)        # segments start on chunk boundaries
    P2, R2 = seg_map(128, T)
    _, S = run_maps(q, k, v, g, beta, S0)
    assert np.allclose(P2 @ (P1 @ S0 + R1) + R2, S, rtol=0, atol=1e-12)


def test_sub_tile_reference_factors_stay_in_range_at_the_decay_bound():
    """g at the bound (every channel -5 on every token): a 64-token cumulative decay
    reaches e^-320, far below fp32, yet the factors the kernels multiply stay finite."""
    q, k, v, g, beta, S0 = inputs(C, 4, 4, seed=3, g_fill=-5.0)
    m = chunk_map(q, k, v, g, beta)
    G, ref = m["G"], m["ref"]
    L = q.shape[0]
    for r in range(L):
        within = np.abs(G[r] - G[ref[r]]).max()           # inside one sub-tile
        assert within <= 5.0 * (ST - 1 - REF) + 1e-9      # at most 8 steps of 5: e^40
        for i in range(L):
            between = G[ref[r]] - G[ref[i]]
            if ref[i] < ref[r]:                           # earlier sub-tile: factor <= 1
                assert (between <= 1e-12).all()
    assert np.isfinite(m["E"]).all()
    o, S = run_maps(q, k, v, g, beta, S0)
    o_ref, S_ref = reference(q, k, v, g, beta, S0)
    assert np.abs(o - o_ref).max() <= 1e-11 * max(1.0, np.abs(o_ref).max())
    assert np.abs(S - S_ref).max() <= 1e-11 * max(1.0, np.abs(S_ref).max())


def _bwd(q, k, v, g, beta, S0, do, dhT):
    """The oracle's gradient on one (sequence, head): (dq, dk, dv, dg, dbeta, dh0)."""
    r = oracle.kda_bwd(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                       beta[None, :, None], S0[None, None], do[None, :, None], dhT[None, None])
    return tuple(x[0, :, 0] for x in r[:5]) + (r[5][0, 0],)


@pytest.mark.parametrize("T,slow", [(150, False), (256, False), (150, True), (256, True)])
def test_state_gradient_chain_over_the_chunk_maps(T, slow):
    """The segmented backward's premise.  With S_out = P S_in + R and O = Q' S_in + O0
    (P = Diag(exp G_C) + M'), the loss is affine in the state at a chunk boundary and
    its gradient there obeys dS_in = Diag(exp G_C) dS_out + M'^T dS_out + Q'^T dO,
    from dS = dL/dhT after the last chunk: the forward update with M'^T for M' and
    Q'^T dO for R, run over the chunks in reverse.  At every boundary it must equal
    the oracle's dL/dh0 of the suffix that starts there.  slow: decays of 0.1-1.1% per
    token, so the state (and its gradient) carries across chunks and the M'^T term
    weighs as much as the others."""
    dk, dv = 12, 10
    q, k, v, g, beta, S0 = inputs(T, dk, dv, seed=T + 5)
    rng = np.random.default_rng(T + 6)
    if slow:
        g = -0.001 - 0.01 * rng.random((T, dk))
    do = rng.standard_normal((T, dv))
    dhT = 0.1 * rng.standard_normal((dk, dv))
    starts = list(range(0, T, C))
    maps = [chunk_map(q[t:t + C], k[t:t + C], v[t:t + C], g[t:t + C], beta[t:t + C])
            for t in starts]
    G = dhT.copy()
    chain = {}
    for t, m in zip(reversed(starts), reversed(maps)):
        G = m["gC"][:, None] * G + m["M"].T @ G + m["Qp"].T @ do[t:t + C]
        chain[t] = G
    for t in starts:
        sl = slice(t, T)
        dh0 = _bwd(q[sl], k[sl], v[sl], g[sl], beta[sl], np.zeros((dk, dv)), do[sl], dhT)[5]
        assert np.abs(chain[t] - dh0).max() <= 1e-10 * max(1.0, np.abs(dh0).max()), t


def test_segments_from_their_boundary_states_and_gradients():
    """The per-token backward run on a segment alone, from the forward state at its
    start and the chain's gradient at its end, gives the whole sequence's gradients
    for the segment's tokens (and, for the first segment, dL/dh0)."""
    T, dk, dv = 200, 8, 6
    q, k, v, g, beta, S0 = inputs(T, dk, dv, seed=31)
    rng = np.random.default_rng(32)
    do = rng.standard_normal((T, dv))
    dhT = 0.1 * rng.standard_normal((dk, dv))
    full = _bwd(q, k, v, g, beta, S0, do, dhT)
    bounds = [0, 64, 128, T]          # segments of whole chunks; the last one ragged
    for a, b in zip(bounds[:-1], bounds[1:]):
        S_a = S0 if a == 0 else reference(q[:a], k[:a], v[:a], g[:a], beta[:a], S0)[1]
        if b == T:
            G_b = dhT
        else:   # dL/dS_b: the suffix's dL/dh0 (the loss is affine in S_b)
            G_b = _bwd(q[b:], k[b:], v[b:], g[b:], beta[b:], np.zeros((dk, dv)), do[b:], dhT)[5]
        part = _bwd(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], S_a, do[a:b], G_b)
        for x, y in zip(part[:5], full[:5]):
            ref = y[a:b]
            assert np.abs(x - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max()), (a, b)
        if a == 0:
            assert np.abs(part[5] - full[5]).max() <= 1e-10 * max(1.0, np.abs(full[5]).max())
