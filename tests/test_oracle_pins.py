"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test names the passage it follows.  Parity status per oracle function:

* ``delta_rule`` (error form)       pinned: worked example, exact recall,
  overwrite recall, reflection parity, closed forms, brute force.
* ``delta_rule`` (transition form)  pinned: agrees with the error form, and
  both with the brute-force expansion.
* ``additive``                      pinned: associative-recall table (additive
  column), overwrite recall at R = 1.
* ``brute_force``                   pinned: worked example, closed forms.
* ``chunked``                       pinned: equals the recurrence at T = 37 for
  chunk sizes 1, 5, 8, 16, 64 with S0 != 0, for all three gates; a planted
  wrong triangle is caught.
* ``wy_transition``                 pinned: equals the explicit product of the
  chunk's transition matrices.
* delta-rule columns of the associative-recall table: parity unpinned (the page
  does not state beta); computed here as context only.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def rand_problem(rng, B, H, T, dk, dv, gate, s0=True, beta_range=(0.05, 1.0)):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    beta = rng.uniform(*beta_range, size=(B, H, T))
    g = None
    if gate == "scalar":
        g = -rng.uniform(0.0, 0.7, size=(B, H, T))
    elif gate == "per_key":
        g = -rng.uniform(0.0, 0.7, size=(B, H, T, dk))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, beta, g, S0


def rel(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


# --- ch. 28, "Correct: the delta rule": the worked example ---------------------

def _worked(d):
    w = gold("worked_example.json")
    k = np.zeros(d); k[: 2] = w["k"]
    q = np.zeros(d); q[: 2] = w["q"]
    v = np.zeros(d); v[: 2] = w["v"]
    betas = [s["beta"] for s in w["steps"]]
    T = len(betas)
    shp = (1, 1, T, d)
    Q = np.broadcast_to(q, shp).copy()
    K = np.broadcast_to(k, shp).copy()
    V = np.broadcast_to(v, shp).copy()
    beta = np.array(betas).reshape(1, 1, T)
    return w, Q, K, V, beta


@pytest.mark.parametrize("d", [2, 64])
def test_worked_example_exact(d):
    w, Q, K, V, beta = _worked(d)
    for form in ("error", "transition"):
        o, S = oracle.delta_rule(Q, K, V, beta, form=form)
        # after both steps: row 0 of the state is exactly v
        assert S[0, 0, 0, :2].tolist() == w["steps"][-1]["state_row0"]
        assert np.all(S[0, 0, 1:] == 0) and np.all(S[0, 0, 0, 2:] == 0)
        for t, st in enumerate(w["steps"]):
            assert o[0, 0, t, :2].tolist() == st["output"], (form, t)
            assert np.all(o[0, 0, t, 2:] == 0)
    # the state after the first step alone
    o1, S1 = oracle.delta_rule(Q[:, :, :1], K[:, :, :1], V[:, :, :1], beta[:, :, :1])
    assert S1[0, 0, 0, :2].tolist() == w["steps"][0]["state_row0"]
    ob, Sb = oracle.brute_force(Q, K, V, beta)
    assert ob[0, 0, :, :2].tolist() == [s["output"] for s in w["steps"]]


# --- ch. 28, "Correct: the delta rule": beta = 1 and a unit key replace the value

@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_exact_single_key_recall(gate):
    rng = np.random.default_rng(11)
    dk, dv, T = 16, 12, 9
    q, k, v, beta, g, S0 = rand_problem(rng, 1, 1, T, dk, dv, gate)
    # keys exactly unit in fp64: basis vectors and a 3-4-5 rational vector
    ks = np.zeros((T, dk))
    for t in range(T):
        if t % 2 == 0:
            ks[t, t % dk] = 1.0
        else:
            ks[t, t % dk] = 0.6
            ks[t, (t + 3) % dk] = 0.8
    k[0, 0] = ks
    beta[:] = 1.0
    # read with q = k: o_t = S_t^T k_t must equal v_t
    o, _ = oracle.delta_rule(k, k, v, beta, g, S0)
    assert rel(o, v) <= 1e-12


# --- D2L 12.5, "Overwriting, measured" ------------------------------------------

def overwrite_recall(rule, R, trials=100, seed=0, d=64, n_keys=8):
    rng = np.random.default_rng(seed + 1000 * R)
    correct = 0
    for _ in range(trials):
        Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
        keys = Qm[:, :n_keys].T                       # 8 orthonormal keys
        vals = rng.standard_normal((n_keys, R, d))
        order = rng.permutation([(i, r) for i in range(n_keys) for r in range(R)])
        # R re-bindings per key, in a shuffled order; the value index r is just a label
        seq_k = np.stack([keys[i] for i, r in order])[None, None]
        seq_v = np.stack([vals[i, r] for i, r in order])[None, None]
        latest = {}
        for i, r in order:
            latest[i] = r
        T = seq_k.shape[2]
        if rule == "delta":
            _, S = oracle.delta_rule(seq_k, seq_k, seq_v, np.ones((1, 1, T)))
        else:
            _, S = oracle.additive(seq_k, seq_k, seq_v)
        S = S[0, 0]
        for i in range(n_keys):
            read = S.T @ keys[i]
            cos = vals[i] @ read / (np.linalg.norm(vals[i], axis=1) * max(np.linalg.norm(read), 1e-300))
            correct += int(np.argmax(cos) == latest[i])
    return correct / (trials * n_keys)


def test_overwrite_recall_table():
    w = gold("overwrite_recall.json")
    prev = None
    for R, want_delta in zip(w["writes_per_key"], w["delta"]):
        assert overwrite_recall("delta", R) == want_delta == 1.0
        add = overwrite_recall("additive", R)
        if R == 1:
            assert add == 1.0
        else:
            assert add < prev
            assert abs(add - 1.0 / R) <= 0.15
        prev = add


# --- D2L 12.5, "One rule, two readings": error form == transition form -----------

@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_error_and_transition_forms_agree(gate):
    rng = np.random.default_rng(3)
    q, k, v, beta, g, S0 = rand_problem(rng, 2, 3, 64, 16, 8, gate)
    o1, S1 = oracle.delta_rule(q, k, v, beta, g, S0, scale=0.7, form="error")
    o2, S2 = oracle.delta_rule(q, k, v, beta, g, S0, scale=0.7, form="transition")
    assert rel(o2, o1) <= 1e-12 and rel(S2, S1) <= 1e-12


def test_forms_agree_at_page_size():
    # the slide's case: d_k = d_v = 64, T = 512, unit keys, beta = sigmoid(N(0,1))
    rng = np.random.default_rng(0)
    T, d = 512, 64
    Q = rng.standard_normal((1, 1, T, d))
    K = rng.standard_normal((1, 1, T, d))
    K /= np.maximum(np.linalg.norm(K, axis=-1, keepdims=True), 1e-12)
    V = rng.standard_normal((1, 1, T, d))
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, 1, T))))
    y1, _ = oracle.delta_rule(Q, K, V, beta, form="error")
    y2, _ = oracle.delta_rule(Q, K, V, beta, form="transition")
    # the page reports 1.38e-06 in fp32 and asserts < 1e-5; fp64 is far tighter
    assert np.abs(y1 - y2).max() / np.abs(y1).max() < 1e-12


# --- explicit expansion on T <= 16 ----------------------------------------------

@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_brute_force_matches_recurrence(gate):
    rng = np.random.default_rng(5)
    q, k, v, beta, g, S0 = rand_problem(rng, 1, 2, 13, 8, 6, gate)
    ob, Sb = oracle.brute_force(q, k, v, beta, g, S0, scale=1.3)
    o, S = oracle.delta_rule(q, k, v, beta, g, S0, scale=1.3)
    assert rel(o, ob) <= 1e-12 and rel(S, Sb) <= 1e-12


# --- special cases with closed forms --------------------------------------------

def test_zero_gate_equals_deltanet_exactly():
    rng = np.random.default_rng(6)
    q, k, v, beta, _, S0 = rand_problem(rng, 2, 2, 40, 16, 16, "none")
    o0, S0_ = oracle.delta_rule(q, k, v, beta, None, S0)
    o1, S1 = oracle.delta_rule(q, k, v, beta, np.zeros(beta.shape), S0)
    assert np.array_equal(o0, o1) and np.array_equal(S0_, S1)


def test_per_key_with_shared_channels_equals_scalar_gate():
    rng = np.random.default_rng(7)
    q, k, v, beta, g, S0 = rand_problem(rng, 2, 2, 40, 16, 16, "scalar")
    gk = np.repeat(g[..., None], 16, axis=-1)
    o1, S1 = oracle.delta_rule(q, k, v, beta, g, S0)
    o2, S2 = oracle.delta_rule(q, k, v, beta, gk, S0)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_beta_zero_is_pure_decay(gate):
    # beta = 0: o_t = (Diag(e^{Gamma_t}) S0)^T (scale q_t) with Gamma_t the inclusive cumsum
    rng = np.random.default_rng(8)
    q, k, v, beta, g, S0 = rand_problem(rng, 1, 2, 20, 8, 8, gate)
    beta[:] = 0.0
    o, S = oracle.delta_rule(q, k, v, beta, g, S0, scale=0.5)
    if g is None:
        lg = np.zeros(k.shape)
    elif g.ndim == 3:
        lg = np.repeat(g[..., None], 8, axis=-1)
    else:
        lg = g
    Gam = np.cumsum(lg, axis=2)
    want = np.einsum("bhtc,bhcj,bhtc->bhtj", np.exp(Gam), S0, 0.5 * q)
    assert rel(o, want) <= 1e-12
    assert rel(S, np.exp(Gam[:, :, -1])[..., None] * S0) <= 1e-12


def test_first_token_from_zero_state():
    # S0 = 0, T = 1: o = beta (scale q . k) v
    rng = np.random.default_rng(9)
    q, k, v, beta, g, _ = rand_problem(rng, 3, 2, 1, 16, 8, "scalar", s0=False)
    o, S = oracle.delta_rule(q, k, v, beta, g, None, scale=0.25)
    want = beta[..., None] * np.sum(0.25 * q * k, -1)[..., None] * v
    assert rel(o, want) <= 1e-13
    assert rel(S, np.einsum("bhc,bhj->bhcj", k[:, :, 0], beta[:, :, 0, None] * v[:, :, 0])) <= 1e-13


# --- D2L 12.5, "The reflection hiding in the delta rule" -------------------------

def test_reflection_eigenvalues():
    w = gold("reflection.json")
    rng = np.random.default_rng(10)
    k = rng.standard_normal(16)
    k /= np.linalg.norm(k)
    for row in w["eigen"]:
        M = oracle.transition_matrix(k, row["beta"], np.zeros(16))
        ev = np.sort(np.linalg.eigvalsh((M + M.T) / 2))
        assert abs(ev[0] - row["along_k"]) < 1e-12 or abs(ev[-1] - row["along_k"]) < 1e-12
        others = ev[1:] if abs(ev[0] - row["along_k"]) < 1e-12 else ev[:-1]
        assert np.allclose(others, row["elsewhere"], atol=1e-12)


@pytest.mark.parametrize("T", [8, 24, 64])
def test_reflection_parity_exact(T):
    # k = e_1, S0 = e_1 e_1^T, v = 0, beta_t = 2 x_t: o_t[0] = (-1)^(x_1 + ... + x_t)
    w = gold("reflection.json")
    rng = np.random.default_rng(T)
    d = 8
    x = rng.integers(0, 2, size=T)
    e1 = np.zeros(d); e1[0] = 1.0
    K = np.broadcast_to(e1, (1, 1, T, d)).copy()
    V = np.zeros((1, 1, T, d))
    S0 = np.zeros((1, 1, d, d)); S0[0, 0, 0, 0] = 1.0
    beta = (2.0 * x).reshape(1, 1, T)
    o, _ = oracle.delta_rule(K, K, V, beta, None, S0)
    want = (-1.0) ** np.cumsum(x)
    acc = float(np.mean(np.sign(o[0, 0, :, 0]) == want))
    assert np.array_equal(o[0, 0, :, 0], want)
    assert acc == w["parity_accuracy_beta2"][str(T)]


# --- ch. 28, "The state is an associative memory": additive column ---------------

def test_associative_recall_additive_column():
    w = gold("associative_recall_64.json")
    d = w["key_dim"]
    rng = np.random.default_rng(12)
    for n, page in zip(w["pairs"], w["additive_error_all"]):
        errs = []
        for _ in range(40):
            K = rng.standard_normal((n, d)); K /= np.linalg.norm(K, axis=1, keepdims=True)
            V = rng.standard_normal((n, d))
            _, S = oracle.additive(K[None, None], K[None, None], V[None, None])
            Rd = K @ S[0, 0]
            errs.append(np.mean(np.linalg.norm(Rd - V, axis=1) / np.linalg.norm(V, axis=1)))
        got = float(np.mean(errs))
        assert abs(got - page) <= 0.10 * page, (n, got, page)
        # and the closed form of the interference: sqrt((n - 1) / d)
        assert abs(got - np.sqrt((n - 1) / d)) <= 0.05 * np.sqrt((n - 1) / d)


# --- ch. 28, "The chunked form": chunked == recurrent, T = 37, S0 != 0 ------------

@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
@pytest.mark.parametrize("chunk", [1, 5, 8, 16, 64])
def test_chunked_matches_recurrence(gate, chunk):
    rng = np.random.default_rng(13)
    q, k, v, beta, g, S0 = rand_problem(rng, 1, 2, 37, 16, 12, gate)
    o, S = oracle.delta_rule(q, k, v, beta, g, S0, scale=0.8)
    oc, Sc = oracle.chunked(q, k, v, beta, g, S0, scale=0.8, chunk=chunk)
    assert rel(oc, o) <= 1e-12 and rel(Sc, S) <= 1e-12


def test_planted_wrong_triangle_is_caught(monkeypatch):
    # ch. 28's note: keeping the wrong triangle of the system passes chunk size 1
    rng = np.random.default_rng(14)
    q, k, v, beta, g, S0 = rand_problem(rng, 1, 1, 37, 16, 12, "scalar")
    o, S = oracle.delta_rule(q, k, v, beta, g, S0)
    monkeypatch.setattr(oracle, "_strict_lower", lambda m: np.tril(m.T, -1))   # transposed coupling
    oc1, _ = oracle.chunked(q, k, v, beta, g, S0, chunk=1)
    oc5, _ = oracle.chunked(q, k, v, beta, g, S0, chunk=5)
    assert rel(oc1, o) <= 1e-12          # chunk size 1 cannot see the mistake
    assert rel(oc5, o) > 1e-3            # a non-divisor chunk size does


# --- D2L 12.5, "Training it: the WY trick" ---------------------------------------

@pytest.mark.parametrize("gate", ["none", "scalar", "per_key"])
def test_wy_transition_equals_explicit_product(gate):
    rng = np.random.default_rng(15)
    C, dk = 10, 12
    _, k, _, beta, g, _ = rand_problem(rng, 1, 1, C, dk, 4, gate)
    k, beta = k[0, 0], beta[0, 0]
    gg = None if g is None else g[0, 0]
    if gg is None:
        lg = np.zeros((C, dk))
    elif gg.ndim == 1:
        lg = np.repeat(gg[:, None], dk, axis=1)
    else:
        lg = gg
    P = np.eye(dk)
    for t in range(C):
        P = oracle.transition_matrix(k[t], beta[t], lg[t]) @ P
    assert rel(oracle.wy_transition(k, beta, gg), P) <= 1e-12


# --- resumability: the state is the checkpoint ------------------------------------

@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_resume_is_exact(gate):
    rng = np.random.default_rng(16)
    q, k, v, beta, g, S0 = rand_problem(rng, 2, 2, 50, 16, 16, gate)
    o, S = oracle.delta_rule(q, k, v, beta, g, S0)
    sl1, sl2 = slice(0, 23), slice(23, 50)
    gp = (lambda s: None) if g is None else (lambda s: g[:, :, s])
    o1, S1 = oracle.delta_rule(q[:, :, sl1], k[:, :, sl1], v[:, :, sl1], beta[:, :, sl1], gp(sl1), S0)
    o2, S2 = oracle.delta_rule(q[:, :, sl2], k[:, :, sl2], v[:, :, sl2], beta[:, :, sl2], gp(sl2), S1)
    assert np.array_equal(np.concatenate([o1, o2], axis=2), o) and np.array_equal(S2, S)


def test_delta_columns_context_only():
    """Delta columns of the 64x64 recall table: parity unpinned (beta not
    stated).  Computed at beta = 1 as context; only sanity-checked: delta's
    error on the last 8 pairs stays below the additive error."""
    d, n = 64, 64
    rng = np.random.default_rng(17)
    K = rng.standard_normal((n, d)); K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((n, d))
    _, S = oracle.delta_rule(K[None, None], K[None, None], V[None, None], np.ones((1, 1, n)))
    _, Sa = oracle.additive(K[None, None], K[None, None], V[None, None])
    last = slice(n - 8, n)
    e_delta = np.mean(np.linalg.norm(K[last] @ S[0, 0] - V[last], axis=1) / np.linalg.norm(V[last], axis=1))
    e_add = np.mean(np.linalg.norm(K[last] @ Sa[0, 0] - V[last], axis=1) / np.linalg.norm(V[last], axis=1))
    assert e_delta < e_add


# ---- the Gated DeltaNet layer's prologue ("The full layer", steps 4 and 5) -----------

def test_gdn_prologue_closed_forms():
    """sigmoid(0) = 1/2; softplus(0) = ln 2 so g = -e^A_log ln 2 at a + dt_bias = 0;
    softplus(x) -> x for large x and -> e^x for very negative x; exp(A_log) scales g."""
    B, H, T, d = 1, 2, 4, 8
    q = np.ones((B, H, T, d)); k = np.ones((B, H, T, d))
    b = np.array([0.0, 2.0, -2.0, 40.0])[None, None].repeat(H, axis=1)
    a = np.array([0.0, 60.0, -60.0, 1.0])[None, None].repeat(H, axis=1)
    A_log = np.array([0.0, np.log(2.0)]); dt_bias = np.zeros(H)
    _, _, beta, g = oracle.gdn_prologue(q, k, b, a, A_log, dt_bias)
    assert beta[0, 0, 0] == 0.5
    assert np.isclose(beta[0, 0, 1], 1 / (1 + np.exp(-2.0)), rtol=0, atol=1e-15)
    assert np.isclose(beta[0, 0, 1] + beta[0, 0, 2], 1.0, rtol=0, atol=1e-15)   # sigmoid(x) + sigmoid(-x) = 1
    assert np.isclose(g[0, 0, 0], -np.log(2.0), rtol=1e-15)
    assert np.isclose(g[0, 1, 0], -2 * np.log(2.0), rtol=1e-15)                   # exp(A_log) = 2
    assert np.isclose(g[0, 0, 1], -60.0, rtol=1e-15)                              # softplus(60) = 60 + e^-60
    assert np.isclose(g[0, 0, 2], -np.exp(-60.0), rtol=1e-12)                     # softplus(-60) ~ e^-60
    assert np.isclose(g[0, 0, 3], -np.log1p(np.e), rtol=1e-15)
    assert (g <= 0).all()


def test_gdn_prologue_dt_bias_shifts_a():
    rng = np.random.default_rng(3)
    a = rng.standard_normal((2, 3, 5)); dtb = rng.standard_normal(3); A_log = rng.standard_normal(3)
    q = rng.standard_normal((2, 3, 5, 4)); b = rng.standard_normal((2, 3, 5))
    g1 = oracle.gdn_prologue(q, q, b, a + dtb[None, :, None], A_log, np.zeros(3))[3]
    g2 = oracle.gdn_prologue(q, q, b, a, A_log, dtb)[3]
    assert np.allclose(g1, g2, rtol=1e-15, atol=0)


def test_gdn_prologue_unit_rows():
    """Unit norm over the head dimension, invariant to a positive scale of the row,
    direction kept; a zero row stays zero (the max(||x||, eps) clamp)."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal((2, 2, 6, 16)); k = rng.standard_normal((2, 2, 6, 16))
    q[0, 0, 0] = 0.0
    b = np.zeros((2, 2, 6)); a = np.zeros((2, 2, 6)); p = np.zeros(2)
    qn, kn, _, _ = oracle.gdn_prologue(q, k, b, a, p, p)
    nq = np.linalg.norm(qn, axis=-1); nk = np.linalg.norm(kn, axis=-1)
    assert np.allclose(nk, 1.0, rtol=0, atol=1e-15)
    assert np.allclose(nq.ravel()[1:], 1.0, rtol=0, atol=1e-15) and nq[0, 0, 0] == 0.0
    qn2, _, _, _ = oracle.gdn_prologue(7.5 * q, k, b, a, p, p)
    assert np.allclose(qn2, qn, rtol=0, atol=1e-15)
    cos = np.sum(qn[0, 1, 2] * q[0, 1, 2]) / np.linalg.norm(q[0, 1, 2])
    assert np.isclose(cos, 1.0, rtol=0, atol=1e-15)


# ---- causal_conv1d: pinned by filters with known outputs, a library convolution and
#      the carried-history property -----------------------------------------------------

def test_causal_conv1d_identity_and_shift_filters():
    """weight [0, .., 0, 1] passes the current input (SiLU of it with the activation);
    weight [1, 0, .., 0] is a delay of K-1 steps that reads the carried state first."""
    rng = np.random.default_rng(11)
    B, T, C, K = 2, 9, 5, 4
    x = rng.standard_normal((B, T, C)); st = rng.standard_normal((B, K - 1, C))
    ident = np.zeros((C, K)); ident[:, K - 1] = 1.0
    y, _ = oracle.causal_conv1d(x, ident, st, activation=False)
    assert np.array_equal(y, x)
    ys, _ = oracle.causal_conv1d(x, ident, st, activation=True)
    assert np.allclose(ys, x / (1 + np.exp(-x)), rtol=1e-15, atol=0)
    delay = np.zeros((C, K)); delay[:, 0] = 1.0
    y, new = oracle.causal_conv1d(x, delay, st, activation=False)
    assert np.array_equal(y[:, :K - 1], st) and np.array_equal(y[:, K - 1:], x[:, :T - K + 1])
    assert np.array_equal(new, x[:, T - K + 1:])
    y0, _ = oracle.causal_conv1d(x, delay, None, activation=False)      # no state: zeros
    assert not y0[:, :K - 1].any()


def test_causal_conv1d_matches_numpy_convolve():
    """Each channel against numpy's full convolution of the joined sequence with the
    reversed filter (the 'valid' part): a library routine the oracle does not use."""
    rng = np.random.default_rng(12)
    B, T, C, K = 2, 13, 6, 4
    x = rng.standard_normal((B, T, C)); w = rng.standard_normal((C, K)); st = rng.standard_normal((B, K - 1, C))
    y, _ = oracle.causal_conv1d(x, w, st, activation=False)
    for b in range(B):
        for c in range(C):
            joined = np.concatenate([st[b, :, c], x[b, :, c]])
            ref = np.convolve(joined, w[c, ::-1], mode="valid")
            assert np.allclose(y[b, :, c], ref, rtol=1e-13, atol=1e-13)


def test_causal_conv1d_impulse_response_and_causality():
    """An impulse at t0 in channel c shows the filter reversed at t0 .. t0+K-1 and
    nothing before t0 or in other channels."""
    B, T, C, K, t0 = 1, 12, 3, 4, 5
    w = np.arange(1.0, C * K + 1).reshape(C, K)
    x = np.zeros((B, T, C)); x[0, t0, 1] = 1.0
    y, _ = oracle.causal_conv1d(x, w, None, activation=False)
    assert not y[0, :t0].any() and not y[0, :, [0, 2]].any()
    assert np.array_equal(y[0, t0:t0 + K, 1], w[1, ::-1])
    assert not y[0, t0 + K:].any()


@pytest.mark.parametrize("T1", [0, 1, 2, 5, 11])
def test_causal_conv1d_carried_state_splits_sequences(T1):
    """Running [0, T1) and then [T1, T) with the returned state equals one run over
    [0, T), including splits shorter than K-1 (the state then keeps old rows)."""
    rng = np.random.default_rng(13 + T1)
    B, T, C, K = 2, 11, 4, 4
    x = rng.standard_normal((B, T, C)); w = rng.standard_normal((C, K)); st = rng.standard_normal((B, K - 1, C))
    y, s = oracle.causal_conv1d(x, w, st)
    ya, sa = oracle.causal_conv1d(x[:, :T1], w, st)
    yb, sb = oracle.causal_conv1d(x[:, T1:], w, sa)
    assert np.allclose(np.concatenate([ya, yb], axis=1), y, rtol=1e-14, atol=1e-14)
    assert np.array_equal(sb, s)


# ---- rms_norm_gated: closed forms --------------------------------------------------------

def test_rms_norm_gated_closed_forms():
    """With eps = 0 the normed row has mean square 1 and is invariant to a positive
    scale of x; a constant row c maps to sign(c); silu(0) = 0 closes the gate;
    sigmoid(0) = 1/2; the weight multiplies channel by channel."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((3, 4, 16)); z = rng.standard_normal((3, 4, 16)); w = rng.standard_normal(16)
    one = np.ones(16)
    big = np.full_like(z, 60.0)          # silu(60) = 60 / (1 + e^-60)
    n = oracle.rms_norm_gated(x, big, one, eps=0.0) / (60.0 / (1 + np.exp(-60.0)))
    assert np.allclose(np.mean(n * n, axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.allclose(oracle.rms_norm_gated(3.7 * x, z, w, eps=0.0), oracle.rms_norm_gated(x, z, w, eps=0.0),
                       rtol=1e-14, atol=1e-14)
    c = np.full((1, 16), -2.5)
    assert np.allclose(oracle.rms_norm_gated(c, big[0, :1], one, eps=0.0), -60.0 / (1 + np.exp(-60.0)), rtol=1e-15)
    assert not oracle.rms_norm_gated(x, np.zeros_like(z), w).any()
    half = oracle.rms_norm_gated(x, np.zeros_like(z), one, eps=0.0, activation="sigmoid")
    assert np.allclose(half, 0.5 * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True)), rtol=1e-14)
    a = oracle.rms_norm_gated(x, z, w); b = oracle.rms_norm_gated(x, z, one)
    assert np.allclose(a, b * w, rtol=1e-14, atol=1e-14)


def test_rms_norm_gated_eps_and_zero_row():
    """eps enters under the root with the mean square: a zero row stays zero and a row
    of rms r is scaled by 1 / sqrt(r^2 + eps)."""
    x = np.zeros((2, 8)); x[1] = 1e-3
    y = oracle.rms_norm_gated(x, np.full((2, 8), 50.0), np.ones(8), eps=1e-6, activation="sigmoid")
    assert not y[0].any()
    expect = 1e-3 / np.sqrt(1e-6 + 1e-6) / (1 + np.exp(-50.0))
    assert np.allclose(y[1], expect, rtol=1e-14)


# ---- generalized_delta_rule: pinned by the ties the page states, a brute-force
#      expansion and the reflection eigenvalues -----------------------------------------------

def _gdr_inputs(B, H, T, dk, dv, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, H, T))))
    S0 = 0.1 * rng.standard_normal((B, H, dk, dv))
    return rng, q, k, v, beta, S0


def test_generalized_rule_tied_is_deltanet():
    """w = 1, kappa = k, a = beta, k_write = beta k: DeltaNet (the page's tie)."""
    rng, q, k, v, beta, S0 = _gdr_inputs(2, 2, 13, 8, 6, 21)
    bk = np.broadcast_to(beta[..., None], k.shape)
    o, S = oracle.generalized_delta_rule(q, np.ones_like(k), k, bk, bk * k, v, S0, scale=0.5)
    o_ref, S_ref = oracle.delta_rule(q, k, v, beta, None, S0, scale=0.5)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12) and np.allclose(S, S_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_generalized_rule_with_decay_is_gated_rule(gate):
    """alpha (I - beta k k^T) with a scalar alpha, and (I - beta k k^T) Diag(alpha)
    with a per-key alpha, are diag(w) - (a * kappa) kappa^T with w = alpha,
    kappa = alpha * k, a = beta / alpha, k_write = beta k."""
    rng, q, k, v, beta, S0 = _gdr_inputs(1, 2, 11, 8, 5, 22)
    if gate == "scalar":
        g = -rng.random((1, 2, 11)); alpha = np.broadcast_to(np.exp(g)[..., None], k.shape)
    else:
        g = -rng.random((1, 2, 11, 8)); alpha = np.exp(g)
    kappa = alpha * k
    a = beta[..., None] / alpha
    o, S = oracle.generalized_delta_rule(q, alpha, kappa, a, beta[..., None] * k, v, S0)
    o_ref, S_ref = oracle.delta_rule(q, k, v, beta, g, S0)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12) and np.allclose(S, S_ref, rtol=0, atol=1e-12)


def test_generalized_rule_brute_force():
    """Explicit products of the d_k x d_k transitions M_t = diag(w_t) - (a_t * kappa_t) kappa_t^T:
    S_t = M_t ... M_1 S0 + sum_s M_t ... M_{s+1} k_write_s v_s^T, with removal and write keys
    unrelated."""
    rng = np.random.default_rng(23)
    T, dk, dv = 6, 5, 4
    q, w, kap, a, kw = (rng.standard_normal((1, 1, T, dk)) for _ in range(5))
    w = 0.5 + 0.5 * np.abs(w)
    v = rng.standard_normal((1, 1, T, dv)); S0 = rng.standard_normal((1, 1, dk, dv))
    o, S = oracle.generalized_delta_rule(q, w, kap, a, kw, v, S0, scale=0.7)
    M = [np.diag(w[0, 0, t]) - np.outer(a[0, 0, t] * kap[0, 0, t], kap[0, 0, t]) for t in range(T)]
    for t in range(T):
        St = S0[0, 0].copy()
        for s in range(t + 1):
            St = M[s] @ St
        for s in range(t + 1):
            P = np.eye(dk)
            for r in range(s + 1, t + 1):
                P = M[r] @ P
            St = St + P @ np.outer(kw[0, 0, s], v[0, 0, s])
        assert np.allclose(o[0, 0, t], 0.7 * St.T @ q[0, 0, t], rtol=0, atol=1e-12 * max(1, np.abs(St).max()))
    assert np.allclose(S[0, 0], St, rtol=0, atol=1e-12 * np.abs(St).max())


def test_generalized_rule_no_removal_is_decayed_sum():
    """a = 0: no removal; the state is the decayed sum of the writes (a closed form)."""
    rng = np.random.default_rng(24)
    T, dk, dv = 9, 4, 3
    w = np.exp(-rng.random((1, 1, T, dk))); kw = rng.standard_normal((1, 1, T, dk))
    v = rng.standard_normal((1, 1, T, dv)); q = rng.standard_normal((1, 1, T, dk))
    _, S = oracle.generalized_delta_rule(q, w, rng.standard_normal((1, 1, T, dk)), np.zeros((1, 1, T, dk)), kw, v)
    ref = sum(np.prod(w[0, 0, s + 1:], axis=0)[:, None] * np.outer(kw[0, 0, s], v[0, 0, s]) for s in range(T))
    assert np.allclose(S[0, 0], ref, rtol=1e-13, atol=1e-14)


def test_generalized_rule_reflection_eigenvalues():
    """With w = 1, a unit kappa and a = beta, the transition is I - beta kappa kappa^T:
    eigenvalue 1 - beta along kappa and 1 elsewhere; the page prints -1 along k at beta = 2.
    The step applied to S = kappa e_1^T shows it (S^T kappa scales by 1 - beta)."""
    fix = gold("reflection.json")
    dk = 6
    kap = np.zeros(dk); kap[2] = 1.0
    for row in fix["eigen"]:
        b = row["beta"]
        S0 = np.zeros((1, 1, dk, 1)); S0[0, 0, :, 0] = kap + np.eye(dk)[4]     # along kappa and orthogonal
        one = np.ones((1, 1, 1, dk))
        _, S = oracle.generalized_delta_rule(np.zeros((1, 1, 1, dk)), one, kap[None, None, None], b * one,
                                             np.zeros((1, 1, 1, dk)), np.zeros((1, 1, 1, 1)), S0)
        assert np.isclose(S[0, 0, 2, 0], row["along_k"], rtol=0, atol=1e-15)
        assert np.isclose(S[0, 0, 4, 0], row["elsewhere"], rtol=0, atol=1e-15)


def test_prologue_two_sigma_gate():
    """allow_neg_eigval doubles the gate: beta = 2 sigmoid(b) in (0, 2), beta(0) = 1."""
    b = np.array([0.0, 3.0, -3.0, 40.0, -40.0])[None, None]
    z = np.zeros((1, 1, 5, 4)); p = np.zeros(1)
    _, _, beta2, _ = oracle.gdn_prologue(z + 1, z + 1, b, b, p, p, allow_neg_eigval=True)
    _, _, beta1, _ = oracle.gdn_prologue(z + 1, z + 1, b, b, p, p)
    assert beta2[0, 0, 0] == 1.0
    assert np.allclose(beta2, 2 * beta1, rtol=1e-15, atol=0)
    assert ((beta2 > 0) & (beta2 <= 2)).all() and np.isclose(beta2[0, 0, 1] + beta2[0, 0, 2], 2.0, rtol=1e-15)


# ---- varlen_delta_rule: pinned by the zero-padding equivalence and by isolation -----------

@pytest.mark.parametrize("gate", [None, "scalar", "per_key"])
def test_varlen_equals_padded_batch(gate):
    """Packing equals a padded batch in which every position past a sequence's end is an
    identity step (beta = 0, g = 0): the padding reading of a partial chunk, applied to
    whole sequences.  Includes an empty sequence."""
    rng = np.random.default_rng(31)
    lens = [5, 0, 11, 1, 7]
    N, H, dk, dv, Tm = len(lens), 2, 6, 4, max(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    Tt = int(cu[-1])
    q = rng.standard_normal((1, H, Tt, dk)); k = rng.standard_normal((1, H, Tt, dk))
    v = rng.standard_normal((1, H, Tt, dv)); beta = 1 / (1 + np.exp(-rng.standard_normal((1, H, Tt))))
    g = None if gate is None else -rng.random((1, H, Tt) if gate == "scalar" else (1, H, Tt, dk))
    S0 = 0.1 * rng.standard_normal((N, H, dk, dv))
    o, ST = oracle.varlen_delta_rule(q, k, v, beta, g, cu, S0, scale=0.3)
    pad = lambda x, tail: np.zeros((N, H, Tm) + tail)
    qp, kp, vp, bp = pad(q, (dk,)), pad(k, (dk,)), pad(v, (dv,)), pad(beta, ())
    gp = None if g is None else pad(g, g.shape[3:])
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        qp[n, :, :b - a], kp[n, :, :b - a], vp[n, :, :b - a], bp[n, :, :b - a] = (
            q[0, :, a:b], k[0, :, a:b], v[0, :, a:b], beta[0, :, a:b])
        if g is not None:
            gp[n, :, :b - a] = g[0, :, a:b]
    op, STp = oracle.delta_rule(qp, kp, vp, bp, gp, S0, scale=0.3)
    assert np.allclose(ST, STp, rtol=0, atol=1e-13)
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        assert np.allclose(o[0, :, a:b], op[n, :, :b - a], rtol=0, atol=1e-13)
    assert np.array_equal(ST[1], S0[1])                 # the empty sequence keeps its state


def test_varlen_sequences_are_isolated():
    """Changing one sequence's tokens or initial state changes nothing in the others."""
    rng = np.random.default_rng(32)
    cu = [0, 4, 9, 16]
    H, dk, dv, Tt = 1, 5, 3, 16
    q, k = rng.standard_normal((1, H, Tt, dk)), rng.standard_normal((1, H, Tt, dk))
    v, beta = rng.standard_normal((1, H, Tt, dv)), 1 / (1 + np.exp(-rng.standard_normal((1, H, Tt))))
    S0 = rng.standard_normal((3, H, dk, dv))
    o1, S1 = oracle.varlen_delta_rule(q, k, v, beta, None, cu, S0)
    v2, S02 = v.copy(), S0.copy()
    v2[:, :, 4:9] += 1.0; S02[1] += 1.0
    o2, S2 = oracle.varlen_delta_rule(q, k, v2, beta, None, cu, S02)
    assert np.array_equal(o1[:, :, :4], o2[:, :, :4]) and np.array_equal(o1[:, :, 9:], o2[:, :, 9:])
    assert np.array_equal(S1[[0, 2]], S2[[0, 2]]) and not np.allclose(S1[1], S2[1])
    with pytest.raises(ValueError):
        oracle.varlen_delta_rule(q, k, v, beta, None, [0, 9, 4, 16], S0)


# ---- gva_delta_rule: pinned by per-head runs, linearity in v and the 1:1 case -------------

def test_gva_value_heads_read_their_key_head():
    """Value head h of a 2-key-head, 6-value-head layer equals a plain one-head run on
    key head h // 3, as the page's repeat_interleave pairs them (not h % 2)."""
    rng = np.random.default_rng(41)
    B, Hk, Hv, T, dk, dv = 2, 2, 6, 9, 5, 4
    q, k = rng.standard_normal((B, Hk, T, dk)), rng.standard_normal((B, Hk, T, dk))
    v = rng.standard_normal((B, Hv, T, dv)); beta = 1 / (1 + np.exp(-rng.standard_normal((B, Hv, T))))
    g = -rng.random((B, Hv, T))
    o, ST = oracle.gva_delta_rule(q, k, v, beta, g, scale=0.4)
    for h in range(Hv):
        oh, sh = oracle.delta_rule(q[:, h // 3:h // 3 + 1], k[:, h // 3:h // 3 + 1], v[:, h:h + 1],
                                   beta[:, h:h + 1], g[:, h:h + 1], scale=0.4)
        assert np.array_equal(o[:, h:h + 1], oh) and np.array_equal(ST[:, h:h + 1], sh)
        if h % Hk != h // 3:
            wrong, _ = oracle.delta_rule(q[:, h % 2:h % 2 + 1], k[:, h % 2:h % 2 + 1], v[:, h:h + 1],
                                         beta[:, h:h + 1], g[:, h:h + 1], scale=0.4)
            assert not np.allclose(o[:, h:h + 1], wrong)


def test_gva_is_linear_in_v_across_shared_heads():
    """Two value heads sharing a key head, with the same beta and g: the rule is linear
    in (v, S0), so their outputs add up to the output for v1 + v2."""
    rng = np.random.default_rng(42)
    B, T, dk, dv = 1, 12, 6, 3
    q, k = rng.standard_normal((B, 1, T, dk)), rng.standard_normal((B, 1, T, dk))
    v = rng.standard_normal((B, 2, T, dv))
    b1 = 1 / (1 + np.exp(-rng.standard_normal((B, 1, T)))); beta = np.repeat(b1, 2, axis=1)
    g1 = -rng.random((B, 1, T)); g = np.repeat(g1, 2, axis=1)
    o, _ = oracle.gva_delta_rule(q, k, v, beta, g)
    osum, _ = oracle.gva_delta_rule(q, k, v.sum(axis=1, keepdims=True), b1, g1)
    assert np.allclose(o.sum(axis=1, keepdims=True), osum, rtol=1e-12, atol=1e-12)


def test_gva_one_to_one_is_the_plain_rule():
    rng = np.random.default_rng(43)
    q, k, v = (rng.standard_normal((1, 3, 7, 4)) for _ in range(3))
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, 3, 7))))
    a, _ = oracle.gva_delta_rule(q, k, v, beta)
    b, _ = oracle.delta_rule(q, k, v, beta)
    assert np.array_equal(a, b)
    with pytest.raises(ValueError):
        oracle.gva_delta_rule(q[:, :2], k[:, :2], v, beta)


@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_chunked_generalized_equals_recurrence(C):
    """The derived chunk algebra of the generalised rule equals the token-by-token rule
    (T = 37, a ragged last chunk, S0 != 0, unrelated removal and write keys)."""
    rng = np.random.default_rng(50 + C)
    B, H, T, dk, dv = 1, 2, 37, 6, 5
    q, kap, kw = (rng.standard_normal((B, H, T, dk)) for _ in range(3))
    kap /= np.linalg.norm(kap, axis=-1, keepdims=True)
    a = rng.random((B, H, T, dk)); w = np.exp(-0.3 * rng.random((B, H, T, dk)))
    v = rng.standard_normal((B, H, T, dv)); S0 = rng.standard_normal((B, H, dk, dv))
    o_ref, S_ref = oracle.generalized_delta_rule(q, w, kap, a, kw, v, S0, scale=0.6)
    o, S = oracle.chunked_generalized(q, w, kap, a, kw, v, S0, scale=0.6, chunk=C)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-11 * np.abs(o_ref).max())
    assert np.allclose(S, S_ref, rtol=0, atol=1e-11 * np.abs(S_ref).max())

