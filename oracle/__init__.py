"""fp64 CPU oracle for the causal delta rule (DeltaNet, Gated DeltaNet, KDA).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never imports, links
or calls anything here, and this package imports nothing from the product.

Contents
--------
``delta_rule``            sequential recurrence in fp64 (C, ``dn_oracle.c``),
                          error form or transition-then-write form.
``additive``              additive (Hebbian) linear attention (C).
``brute_force``           explicit expansion with d_k x d_k products, T <= 16.
``chunked``               fp64 restatement of the chunkwise (UT transform)
                          equations, used only to check the chunk algebra
                          against the sequential recurrence.
``wy_transition``         the WY form of one chunk's product of transitions.
``gdn_prologue``          steps 4 and 5 of the Gated DeltaNet layer: unit q and
                          k, beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias).
``causal_conv1d``        step 2 of the layer: depthwise causal conv over time
                          (kernel K, SiLU) with the K-1 previous inputs carried.
``rms_norm_gated``        step 7 of the layer: RMSNorm of each head's output
                          times a per-channel weight and SiLU (or sigmoid) of z.
``generalized_delta_rule`` RWKV-7's form: per-channel decay, removal key and
                          rate, and a separate write key.
``chunked_generalized``   its chunkwise form (derived; checks the chunk algebra).
``varlen_delta_rule``     sequences packed along time (cu_seqlens), each with
                          its own initial and final state.
``gva_delta_rule``        grouped value heads: H_v / H_k value heads share each
                          key head's q and k.

Every function takes and returns numpy arrays.  Layouts: tokens
``[B, H, T, d]``, beta and a scalar gate ``[B, H, T]``, a per-key gate
``[B, H, T, d_k]``, states ``[B, H, d_k, d_v]`` (row i = key channel).
The gate argument ``g`` is the log-decay; the decay is ``exp(g)``.

Pins: see ``tests/test_oracle_pins.py``.  Parity status of each function is
listed there; the delta-rule columns of the 64x64 associative-recall table in
"Linear attention and Gated DeltaNet" (ch. 28, "The state is an associative
memory") are parity unpinned (the page does not state beta), every other
function here is pinned.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

GATE_NONE, GATE_SCALAR, GATE_PER_KEY = 0, 1, 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        L = ctypes.c_long
        for name in ("dno_delta_error_form", "dno_delta_transition_form"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, dp, dp, dp,
                           L, L, L, L, L, ctypes.c_double, ctypes.c_int]
        lib.dno_additive.restype = ctypes.c_int
        lib.dno_additive.argtypes = [dp, dp, dp, dp, dp, dp, L, L, L, L, L,
                                     ctypes.c_double, ctypes.c_int]
        lib.dno_max_threads.restype = ctypes.c_int
        lib.dno_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the C oracle uses when ``nthreads=0`` (OpenMP default)."""
    return int(_load().dno_max_threads())


def _f64(x):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gate_kind(g, k) -> int:
    """Infer the gate from the shape of ``g``: None, [B,H,T] or [B,H,T,d_k]."""
    if g is None:
        return GATE_NONE
    g = np.asarray(g)
    if g.shape == np.asarray(k).shape[:-1]:
        return GATE_SCALAR
    if g.shape == np.asarray(k).shape:
        return GATE_PER_KEY
    raise ValueError(f"gate shape {g.shape} matches neither [B,H,T] nor [B,H,T,d_k]")


def delta_rule(q, k, v, beta, g=None, S0=None, scale=1.0, form="error",
               nthreads=0):
    """Run the delta rule token by token in fp64; return ``(o, S_T)``.

    ``form="error"``: forget, predict, correct, write, read ("Linear attention
    and Gated DeltaNet", ch. 28, "Gated DeltaNet" and "The recurrent form";
    KDA per "A walk through of the DeltaNet family", its KDA update).
    ``form="transition"``: ``S = (I - beta k k^T) Diag(alpha) S + beta k v^T``
    with an explicit d_k x d_k matrix (D2L 12.5, "One rule, two readings",
    matrix form; "Gating: the modern cell").
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    gate = gate_kind(g, k)
    g = _f64(g)
    S0 = _f64(S0)
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape[:3] == (B, H, T) and beta.shape == (B, H, T)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.empty((B, H, T, dv), np.float64)
    ST = np.empty((B, H, dk, dv), np.float64)
    fn = {"error": _load().dno_delta_error_form,
          "transition": _load().dno_delta_transition_form}[form]
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), gate, _ptr(S0),
            _ptr(o), _ptr(ST), B, H, T, dk, dv, float(scale), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, ST


def additive(q, k, v, S0=None, scale=1.0, nthreads=0):
    """Additive linear attention ``S += k v^T``, ``o = S^T (scale q)`` in fp64
    ("Linear attention and Gated DeltaNet", ch. 28, "Removing the softmax")."""
    q, k, v, S0 = _f64(q), _f64(k), _f64(v), _f64(S0)
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    o = np.empty((B, H, T, dv), np.float64)
    ST = np.empty((B, H, dk, dv), np.float64)
    rc = _load().dno_additive(_ptr(q), _ptr(k), _ptr(v), _ptr(S0), _ptr(o),
                              _ptr(ST), B, H, T, dk, dv, float(scale),
                              int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, ST


# ---------------------------------------------------------------------------
# numpy restatements (fp64), written from the displayed equations
# ---------------------------------------------------------------------------

def _decay_vectors(g, k):
    """Per-token, per-key-channel log-decay ``[B,H,T,d_k]``: zeros without a
    gate, the scalar broadcast over channels for Gated DeltaNet, itself for
    KDA.  With identical channels the per-key formulas below are exactly the
    scalar ones."""
    k = np.asarray(k)
    gate = gate_kind(g, k)
    if gate == GATE_NONE:
        return np.zeros(k.shape, np.float64)
    g = np.asarray(g, np.float64)
    if gate == GATE_SCALAR:
        return np.broadcast_to(g[..., None], k.shape).astype(np.float64)
    return g.copy()


def transition_matrix(k_t, beta_t, logdecay_t):
    """``M_t = (I - beta_t k_t k_t^T) Diag(exp(logdecay_t))`` (d_k x d_k): the
    per-token transition of the delta rule, forget first (D2L 12.5, "Gating:
    the modern cell"; KDA order per "A walk through of the DeltaNet family")."""
    k_t = np.asarray(k_t, np.float64)
    dk = k_t.shape[0]
    return (np.eye(dk) - beta_t * np.outer(k_t, k_t)) * np.exp(logdecay_t)[None, :]


def brute_force(q, k, v, beta, g=None, S0=None, scale=1.0):
    """Explicit expansion, no recursion on S (T <= 16):

        S_t = (M_t ... M_1) S_0 + sum_{j<=t} (M_t ... M_{j+1}) beta_j k_j v_j^T
        o_t = S_t^T (scale q_t)

    Every product is formed afresh from the transition matrices."""
    q, k, v, beta = (np.asarray(x, np.float64) for x in (q, k, v, beta))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    if T > 16:
        raise ValueError("brute force expansion is for T <= 16")
    lg = _decay_vectors(g, k)
    S0 = np.zeros((B, H, dk, dv)) if S0 is None else np.asarray(S0, np.float64)
    o = np.empty((B, H, T, dv))
    ST = np.empty((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            Ms = [transition_matrix(k[b, h, t], beta[b, h, t], lg[b, h, t]) for t in range(T)]

            def prod(hi, lo):  # M_hi ... M_lo  (1-based, inclusive); identity if lo > hi
                P = np.eye(dk)
                for s in range(lo, hi + 1):
                    P = Ms[s - 1] @ P
                return P

            for t in range(1, T + 1):
                S = prod(t, 1) @ S0[b, h]
                for j in range(1, t + 1):
                    S = S + prod(t, j + 1) @ (beta[b, h, j - 1] * np.outer(k[b, h, j - 1], v[b, h, j - 1]))
                o[b, h, t - 1] = S.T @ (scale * q[b, h, t - 1])
                if t == T:
                    ST[b, h] = S
            if T == 0:
                ST[b, h] = S0[b, h]
    return o, ST


def _strict_lower(m):
    """Entries strictly below the diagonal (the chunk system's coupling)."""
    return np.tril(m, -1)


def _lower(m):
    """Entries on and below the diagonal (causal mask, diagonal kept)."""
    return np.tril(m, 0)


def _solve_unit_lower(L, rhs):
    """Solve ``L X = rhs`` for unit lower-triangular L (a library routine)."""
    from scipy.linalg import solve_triangular
    return solve_triangular(L, rhs, lower=True, unit_diagonal=True)


def chunked(q, k, v, beta, g=None, S0=None, scale=1.0, chunk=64):
    """Chunkwise form in fp64, from the displayed equations of "Linear
    attention and Gated DeltaNet" (ch. 28, "The chunked form: recurrence as
    matrix multiplication"), extended to a per-key decay.

    The sequence is zero-padded to a multiple of ``chunk`` (q, k, v rows zero,
    beta = 0 and log-decay 0, i.e. identity steps) and split into chunks.
    Inside a chunk, with Gamma_i = sum_{m<=i} g_m (per key channel),
    kd_ij = sum_c k_ic k_jc exp(Gamma_ic - Gamma_jc) and
    qd_ij = sum_c q_ic k_jc exp(Gamma_ic - Gamma_jc) for j <= i:

        (I + strict_tril(beta_i kd_ij)) U = beta V - beta (K * e^Gamma) S_0
        O     = (Q * e^Gamma) S_0 + tril(qd) U
        S_end = Diag(e^Gamma_C) S_0 + (K * e^(Gamma_C - Gamma))^T U

    With one decay shared by every channel these are the page's equations
    with D_ij = exp(G_i - G_j).  ``scale`` multiplies q before anything else.
    """
    q, k, v, beta = (np.asarray(x, np.float64) for x in (q, k, v, beta))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    lg = _decay_vectors(g, k)
    q = q * scale
    C = int(chunk)
    pad = (-T) % C
    if pad:
        q = np.concatenate([q, np.zeros((B, H, pad, dk))], axis=2)
        k = np.concatenate([k, np.zeros((B, H, pad, dk))], axis=2)
        v = np.concatenate([v, np.zeros((B, H, pad, dv))], axis=2)
        beta = np.concatenate([beta, np.zeros((B, H, pad))], axis=2)
        lg = np.concatenate([lg, np.zeros((B, H, pad, dk))], axis=2)
    n = (T + pad) // C
    S_all = np.zeros((B, H, dk, dv)) if S0 is None else np.array(S0, np.float64)
    out = np.zeros((B, H, T + pad, dv))
    for b in range(B):
        for h in range(H):
            S = S_all[b, h].copy()
            for c in range(n):
                sl = slice(c * C, (c + 1) * C)
                Qc, Kc, Vc = q[b, h, sl], k[b, h, sl], v[b, h, sl]
                bc = beta[b, h, sl]
                Gam = np.cumsum(lg[b, h, sl], axis=0)            # [C, dk], inclusive
                # pairwise decayed products, j <= i only (upper part is masked)
                diff = Gam[:, None, :] - Gam[None, :, :]          # [i, j, c]
                causal = np.tril(np.ones((C, C), bool))
                Dp = np.where(causal[..., None], np.exp(np.where(causal[..., None], diff, 0.0)), 0.0)
                kd = np.einsum("ic,jc,ijc->ij", Kc, Kc, Dp)
                qd = np.einsum("ic,jc,ijc->ij", Qc, Kc, Dp)
                system = np.eye(C) + _strict_lower(bc[:, None] * kd)
                rhs = bc[:, None] * Vc - bc[:, None] * ((Kc * np.exp(Gam)) @ S)
                U = _solve_unit_lower(system, rhs)
                out[b, h, sl] = (Qc * np.exp(Gam)) @ S + _lower(qd) @ U
                tail = np.exp(Gam[-1][None, :] - Gam)             # [C, dk]
                S = np.exp(Gam[-1])[:, None] * S + (Kc * tail).T @ U
            S_all[b, h] = S
    return out[:, :, :T], S_all


def wy_transition(k, beta, g=None):
    """Product of one chunk's transitions ``M_C ... M_1`` in WY form:

        Diag(e^Gamma_C) - (K * e^(Gamma_C - Gamma))^T W,
        W = (I + strict_tril(beta_i kd_ij))^{-1} (beta * K * e^Gamma)

    for a single chunk: ``k [C, d_k]``, ``beta [C]``, ``g`` None, ``[C]`` or
    ``[C, d_k]`` (D2L 12.5, "Training it: the WY trick"; ch. 28's chunk
    system, whose S_0-dependent part this is)."""
    k = np.asarray(k, np.float64)
    beta = np.asarray(beta, np.float64)
    C, dk = k.shape
    lg = _decay_vectors(None if g is None else np.asarray(g)[None, None],
                        k[None, None])[0, 0]
    Gam = np.cumsum(lg, axis=0)
    kd = np.zeros((C, C))
    for i in range(C):
        for j in range(i + 1):
            kd[i, j] = np.sum(k[i] * k[j] * np.exp(Gam[i] - Gam[j]))
    system = np.eye(C) + _strict_lower(beta[:, None] * kd)
    W = _solve_unit_lower(system, beta[:, None] * k * np.exp(Gam))
    return np.diag(np.exp(Gam[-1])) - (k * np.exp(Gam[-1][None, :] - Gam)).T @ W


def gdn_prologue(q, k, b, a, A_log, dt_bias, eps=1e-12, allow_neg_eigval=False):
    """Steps 4 and 5 of the Gated DeltaNet layer ("Linear attention and Gated
    DeltaNet", ch. 28, "The full layer"), in fp64, on raw per-token inputs:

    - q and k normalised over the head dimension, x / max(||x||_2, eps): the
      pages call l2norm without defining it and elsewhere use the
      F.normalize contract for unit keys, which this restates;
    - beta = sigmoid(b), the write strength in (0, 1); with allow_neg_eigval,
      beta = 2 sigmoid(b) in (0, 2), so that I - beta k k^T can have a negative
      eigenvalue along k ("DeltaNet: Memory That Edits", "The reflection
      hiding in the delta rule");
    - g = -exp(A_log[h]) * softplus(a + dt_bias[h]), the log-decay (always
      negative), with softplus(x) = log(1 + e^x) (numpy's logaddexp(0, x)).

    q, k [B,H,T,d_k]; b, a [B,H,T]; A_log, dt_bias [H].  Returns
    ``(q_hat, k_hat, beta, g)``; ``scale`` still applies to q_hat inside the
    rule."""
    q, k, b, a = _f64(q), _f64(k), _f64(b), _f64(a)
    A_log, dt_bias = _f64(A_log), _f64(dt_bias)
    qn = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), eps)
    kn = k / np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), eps)
    beta = (2.0 if allow_neg_eigval else 1.0) / (1.0 + np.exp(-b))
    g = -np.exp(A_log)[None, :, None] * np.logaddexp(0.0, a + dt_bias[None, :, None])
    return qn, kn, beta, g


def causal_conv1d(x, weight, state=None, activation=True):
    """Step 2 of the Gated DeltaNet layer ("Linear attention and Gated
    DeltaNet", ch. 28, "The full layer" and its ``causal_conv1d``), in fp64:
    a depthwise causal convolution over time, one length-K filter per channel,
    then SiLU, carrying the previous K-1 inputs as its state.

    Written from its definition: with ``joined = concat(state, x)`` along time
    (K-1 history rows, then the T new rows),

        y[t, c] = sum_{j=0}^{K-1} weight[c, j] * joined[t + j, c],

    so ``weight[c, K-1]`` multiplies the current input and output t sees
    inputs t-K+1 .. t only; ``silu(y) = y / (1 + e^-y)`` when ``activation``.
    The new state is the last K-1 rows of ``joined``.

    Layout: token-major, x [B, T, C] and state [B, K-1, C] (oldest row
    first); the page writes the same arrays channel-major.  weight [C, K].
    A missing state is K-1 rows of zeros.  Returns ``(y, new_state)``."""
    x, weight = _f64(x), _f64(weight)
    B, T, C = x.shape
    K = weight.shape[1]
    state = np.zeros((B, K - 1, C)) if state is None else _f64(state)
    joined = np.concatenate([state, x], axis=1)
    y = np.zeros((B, T, C))
    for t in range(T):
        for j in range(K):
            y[:, t, :] += weight[:, j][None, :] * joined[:, t + j, :]
    if activation:
        y = y / (1.0 + np.exp(-y))
    return y, joined[:, T:, :].copy()


def rms_norm_gated(x, z, weight, eps=1e-6, activation="silu"):
    """Step 7 of the Gated DeltaNet layer ("Linear attention and Gated
    DeltaNet", ch. 28, ``RMSNormGated``), in fp64: each row of a head's
    read-out divided by its root mean square, times a per-channel weight and
    a gate of z,

        y = weight * x / sqrt(mean(x^2) + eps) * act(z),

    act = SiLU (``z / (1 + e^-z)``) or the logistic sigmoid.  The mean runs
    over the last axis (the head's d_v channels); weight [d_v] is shared by
    every head.  x and z have the same shape; returns y of that shape."""
    x, z, weight = _f64(x), _f64(z), _f64(weight)
    normed = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if activation == "silu":
        gate = z / (1.0 + np.exp(-z))
    elif activation == "sigmoid":
        gate = 1.0 / (1.0 + np.exp(-z))
    else:
        raise ValueError(f"activation {activation!r}")
    return weight * normed * gate


def generalized_delta_rule(q, w, kappa, a, k_write, v, S0=None, scale=1.0):
    """The generalised delta rule of RWKV-7 ("DeltaNet: Memory That Edits",
    "The generalized delta rule"), token by token in fp64:

        S_t = (diag(w_t) - (a_t * kappa_t) kappa_t^T) S_{t-1} + k_write_t v_t^T,
        o_t = S_t^T (scale q_t),

    with a per-channel decay w_t, a removal key kappa_t, a per-channel removal
    rate a_t and a write key k_write_t that need not equal kappa_t.  The page
    writes the state in the d_k x d_v orientation used here; the read-out
    through q follows the rest of the family (o = S^T q).  Tying them,
    w = 1, kappa = k, a = beta, k_write = beta k, gives DeltaNet.

    q, w, kappa, a, k_write [B,H,T,d_k]; v [B,H,T,d_v]; S0 [B,H,d_k,d_v] or
    None.  Returns ``(o, S_T)``."""
    q, w, kappa, a, k_write, v = (_f64(x) for x in (q, w, kappa, a, k_write, v))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, H, T, dv))
    for t in range(T):
        removed = np.einsum("bhk,bhkv->bhv", kappa[:, :, t], S)             # kappa^T S
        S = (w[:, :, t, :, None] * S
             - (a[:, :, t] * kappa[:, :, t])[..., None] * removed[:, :, None, :]
             + k_write[:, :, t, :, None] * v[:, :, t, None, :])
        o[:, :, t] = scale * np.einsum("bhkv,bhk->bhv", S, q[:, :, t])
    return o, S


def varlen_delta_rule(q, k, v, beta, g, cu_seqlens, S0=None, scale=1.0):
    """Variable-length packing ("Linear attention and Gated DeltaNet", ch. 28,
    "The state a request carries": every request carries its own fixed-size
    state): N sequences packed along time, sequence n holding tokens
    cu_seqlens[n] .. cu_seqlens[n+1]-1, each run by ``delta_rule`` from its own
    initial state and yielding its own final state.

    q, k [1,H,T_total,d_k]; v [1,H,T_total,d_v]; beta and a scalar g
    [1,H,T_total], a per-key g [1,H,T_total,d_k], or None; cu_seqlens [N+1]
    non-decreasing from 0 to T_total; S0 [N,H,d_k,d_v] or None.  Returns
    ``(o [1,H,T_total,d_v], S_T [N,H,d_k,d_v])``."""
    cu = [int(c) for c in cu_seqlens]
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    g = _f64(g)
    _, H, T, dk = k.shape
    dv = v.shape[-1]
    if cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must rise from 0 to T_total")
    N = len(cu) - 1
    o = np.zeros((1, H, T, dv))
    ST = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        s0 = None if S0 is None else _f64(S0)[n:n + 1]
        if b == a:
            ST[n] = 0.0 if s0 is None else s0[0]
            continue
        gn = None if g is None else g[:, :, a:b]
        o[:, :, a:b], st = delta_rule(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], beta[:, :, a:b], gn, s0,
                                      scale=scale)
        ST[n] = st[0]
    return o, ST


def gva_delta_rule(q, k, v, beta, g=None, S0=None, scale=1.0):
    """Grouped value heads ("Linear attention and Gated DeltaNet", ch. 28, "The
    full layer", step 3): more value heads than key heads, each key head shared
    by H_v / H_k consecutive value heads, so that value head h reads q and k of
    key head h // (H_v / H_k) (the layer's repeat_interleave of q and k over the
    head axis).  beta, g and the state belong to the value heads.

    q, k [B,H_k,T,d_k]; v [B,H_v,T,d_v]; beta [B,H_v,T]; g None, [B,H_v,T] or
    [B,H_v,T,d_k]; S0 [B,H_v,d_k,d_v] or None.  Returns ``(o [B,H_v,T,d_v],
    S_T [B,H_v,d_k,d_v])``."""
    q, k = _f64(q), _f64(k)
    Hk, Hv = k.shape[1], v.shape[1]
    if Hv % Hk != 0:
        raise ValueError("the value heads must be a multiple of the key heads")
    r = Hv // Hk
    return delta_rule(np.repeat(q, r, axis=1), np.repeat(k, r, axis=1), v, beta, g, S0, scale=scale)


def chunked_generalized(q, w, kappa, a, k_write, v, S0=None, scale=1.0, chunk=64):
    """Chunkwise form of ``generalized_delta_rule`` in fp64, derived here from
    the recurrence (the page gives only the recurrence): used only to check
    the chunk algebra a chunked kernel would use against the token-by-token
    rule.  Within a chunk, with l_s = a_s * kappa_s (left removal vector),
    r_s = kappa_s (right), G_t = sum_{s<=t} log w_s per channel (chunk-local,
    G_0 = 0) and U_s = r_s^T S_{s-1} (the removed content):

        (I + M) U = R S_0 + N V,
        M_sj = r_s^T e^(G_{s-1} - G_j) l_j,  N_sj = r_s^T e^(G_{s-1} - G_j) kw_j   (j < s),
        R_s  = r_s^T e^(G_{s-1}),
        S_C  = e^(G_C) S_0 + sum_s e^(G_C - G_s) (kw_s v_s^T - l_s U_s),
        o_t  = scale (q_t^T e^(G_t) S_0 + sum_{s<=t} q_t^T e^(G_t - G_s) (kw_s v_s^T - l_s U_s)).

    Explicit pairwise decays and a library triangular solve; w must be
    positive.  Same arguments and result as ``generalized_delta_rule``."""
    q, w, kappa, a, kw, v = (_f64(x) for x in (q, w, kappa, a, k_write, v))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
    o = np.zeros((B, H, T, dv))
    for b in range(B):
        for h in range(H):
            St = S[b, h]
            for c0 in range(0, T, chunk):
                sl = slice(c0, min(c0 + chunk, T))
                Q, L, Rv, Kw, V = q[b, h, sl], a[b, h, sl] * kappa[b, h, sl], kappa[b, h, sl], kw[b, h, sl], v[b, h, sl]
                G = np.cumsum(np.log(w[b, h, sl]), axis=0)                 # G_1 .. G_C
                n = G.shape[0]
                Gp = np.vstack([np.zeros((1, dk)), G[:-1]])                # G_{s-1}
                M = np.zeros((n, n)); N = np.zeros((n, n))
                for s_ in range(n):
                    for j in range(s_):
                        dec = np.exp(Gp[s_] - G[j])
                        M[s_, j] = np.sum(Rv[s_] * dec * L[j])
                        N[s_, j] = np.sum(Rv[s_] * dec * Kw[j])
                R = Rv * np.exp(Gp)
                U = _solve_unit_lower(np.eye(n) + M, R @ St + N @ V)
                W = Kw[:, :, None] * V[:, None, :] - L[:, :, None] * U[:, None, :]     # per s: kw v^T - l U
                for t in range(n):
                    dec = np.exp(G[t][None, :] - G[:t + 1])                  # e^(G_t - G_s), s <= t
                    St_t = np.exp(G[t])[:, None] * St + np.einsum("sk,skv->kv", dec, W[:t + 1])
                    o[b, h, c0 + t] = scale * St_t.T @ Q[t]
                dec = np.exp(G[-1][None, :] - G)
                St = np.exp(G[-1])[:, None] * St + np.einsum("sk,skv->kv", dec, W)
            S[b, h] = St
    return o, S
