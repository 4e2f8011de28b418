"""The chunk identities behind the layer-prologue kernels, in fp64 on the CPU.

The tensor-core prefill with the Gated DeltaNet layer's prologue fused in
("Linear attention and Gated DeltaNet", ch. 28, "The full layer", steps 4
and 5) never writes unit q and k.  It keeps the raw tiles and carries the
norms as per-row factors r_q = 1/||q_i|| and r_k = 1/||k_i||.  These tests
check two placements of those factors against the sequential recurrence (the
oracle) run on the normalised inputs, over several chunks with a carried
state:

- the plain placement:
  - A_ij carries r_ki r_kj, and P_ij carries r_qi r_kj;
  - W = T diag(beta e^G r_k) K;
  - Q-hat rows carry r_q, and the rows of U~ carry r_k;
- the kernels' placement, a fold that keeps r_k out of the state pass:
  u' = diag(r_k) u, W' = diag(r_k) W and P' = P diag(1/r_k) (rows still
  carrying r_q), so that U' = u' - W'S = diag(r_k) U, K^T U~' = K-hat^T U~
  and P'U' = PU; Q-hat keeps its r_q, and the output rows need no factor;
- the full fold, which also moves r_q to the output rows: P'' = scale tril(QK^T * D),
  with no norm factor at all, Q-hat without r_q, and O = diag(r_q)(Q-hat S + P''U').

The chunk equations are those of the chunked form on the same page (A, T,
W, u, P; U = u - WS; O = Q-hat S + PU; S <- e^(G_last) S + K~^T U)."""
import numpy as np
import pytest

import oracle


def chunk_pass(q, k, v, beta, g, S0, scale, C, fold, drop_rk_on_u=False):
    """One (b, h) through chunks of C with the prologue's factors placed as the
    kernels place them (fold=False), with r_k folded into u, W and P
    (fold=True), or with r_q moved to the output rows as well (fold="all").
    drop_rk_on_u plants a mistake: the rows of U~ lose their r_k."""
    T = k.shape[0]
    rq = 1.0 / np.maximum(np.linalg.norm(q, axis=1), 1e-12)
    rk = 1.0 / np.maximum(np.linalg.norm(k, axis=1), 1e-12)
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        Q, K, V, b, G = q[sl], k[sl], v[sl], beta[sl], np.cumsum(g[sl])
        r_q, r_k = rq[sl], rk[sl]
        n = K.shape[0]
        D = np.tril(np.exp(G[:, None] - G[None, :]))
        A = np.tril((b * r_k)[:, None] * (K @ K.T) * D * r_k[None, :], -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ ((b * np.exp(G) * r_k)[:, None] * K)
        u = Tm @ (b[:, None] * V)
        P = scale * np.tril(r_q[:, None] * (Q @ K.T) * D * r_k[None, :])
        Qh = (scale * np.exp(G) * r_q)[:, None] * Q
        decay = np.exp(G[-1] - G)
        if not fold:
            U = u - W @ S
            o[sl] = Qh @ S + P @ U
            row = decay if drop_rk_on_u else decay * r_k
            S = np.exp(G[-1]) * S + K.T @ (row[:, None] * U)
        elif fold is True:
            u2, W2 = r_k[:, None] * u, r_k[:, None] * W
            P2 = P / r_k[None, :]
            U2 = u2 - W2 @ S
            o[sl] = Qh @ S + P2 @ U2
            S = np.exp(G[-1]) * S + K.T @ (decay[:, None] * U2)
        else:
            u2, W2 = r_k[:, None] * u, r_k[:, None] * W
            P3 = scale * np.tril((Q @ K.T) * D)                 # the plain path's P
            Qh3 = (scale * np.exp(G))[:, None] * Q                # the plain path's Q-hat
            U2 = u2 - W2 @ S
            o[sl] = r_q[:, None] * (Qh3 @ S + P3 @ U2)
            S = np.exp(G[-1]) * S + K.T @ (decay[:, None] * U2)
    return o, S


def layer_case(T, seed, dk=16, dv=12):
    rng = np.random.default_rng(seed)
    q = 3 * rng.standard_normal((T, dk)); k = 3 * rng.standard_normal((T, dk)); v = rng.standard_normal((T, dv))
    b = rng.standard_normal(T); a = rng.standard_normal(T)
    A_log, dt_bias = np.array([0.3]), np.array([-0.2])
    S0 = 0.1 * rng.standard_normal((dk, dv))
    qn, kn, beta, g = oracle.gdn_prologue(q[None, None], k[None, None], b[None, None], a[None, None], A_log, dt_bias)
    return q, k, v, beta[0, 0], g[0, 0], S0, qn, kn


@pytest.mark.parametrize("fold", [False, True, "all"])
@pytest.mark.parametrize("T,C", [(37, 8), (64, 16), (50, 64)])
def test_prologue_factor_placement_matches_recurrence(fold, T, C):
    q, k, v, beta, g, S0, qn, kn = layer_case(T, 100 + T + C)
    scale = q.shape[1] ** -0.5
    o_ref, S_ref = oracle.delta_rule(qn, kn, v[None, None], beta[None, None], g[None, None], S0[None, None],
                                     scale=scale)
    o, S = chunk_pass(q, k, v, beta, g, S0, scale, C, fold)
    assert np.allclose(o, o_ref[0, 0], rtol=0, atol=1e-12 * np.abs(o_ref).max())
    assert np.allclose(S, S_ref[0, 0], rtol=0, atol=1e-12 * np.abs(S_ref).max())


def test_factor_placement_catches_a_dropped_factor():
    """The check is not vacuous: the same pass with r_k left off the rows of U~
    misses the recurrence by far more than rounding."""
    q, k, v, beta, g, S0, qn, kn = layer_case(40, 7)
    o_ref, S_ref = oracle.delta_rule(qn, kn, v[None, None], beta[None, None], g[None, None], S0[None, None])
    o, S = chunk_pass(q, k, v, beta, g, S0, 1.0, 8, fold=False, drop_rk_on_u=True)
    assert np.abs(S - S_ref[0, 0]).max() > 1e-3 * np.abs(S_ref).max()
    assert np.abs(o - o_ref[0, 0]).max() > 1e-3 * np.abs(o_ref).max()


@pytest.mark.parametrize("fold", [True, "all"])
def test_fold_with_zero_rows(fold):
    """A zero key row gets r_k = 1e12 and a zero query row r_q = 1e12 (the
    max(||x||, 1e-12) clamp).  The fold then scales u and W rows by 1e12, and
    still matches the recurrence, whose unit key and query are zero there."""
    q, k, v, beta, g, S0, qn, kn = layer_case(30, 11)
    q[3] = 0.0; k[5] = 0.0; k[17] = 0.0
    qn, kn, _, _ = oracle.gdn_prologue(q[None, None], k[None, None], np.zeros((1, 1, 30)), np.zeros((1, 1, 30)),
                                       np.zeros(1), np.zeros(1))
    scale = q.shape[1] ** -0.5
    o_ref, S_ref = oracle.delta_rule(qn, kn, v[None, None], beta[None, None], g[None, None], S0[None, None],
                                     scale=scale)
    o, S = chunk_pass(q, k, v, beta, g, S0, scale, 8, fold)
    assert np.isfinite(o).all() and np.isfinite(S).all()
    assert np.allclose(o, o_ref[0, 0], rtol=0, atol=1e-9 * np.abs(o_ref).max())
    assert np.allclose(S, S_ref[0, 0], rtol=0, atol=1e-9 * np.abs(S_ref).max())
    assert not o[3].any() or np.abs(o[3]).max() <= 1e-9 * np.abs(o_ref).max()
