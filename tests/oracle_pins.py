"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics.

Each ``pin_*`` takes a loaded oracle library and raises AssertionError when the
oracle disagrees with something that does not depend on the oracle itself:
closed forms, a separately written scalar-gate (Gated DeltaNet) recurrence,
library routines (torch's CPU conv1d, numpy norms), and structural identities.
``test_oracle_pins.py`` runs them on the real oracle and on deliberately broken
copies of it, to show that each plausible mistake is caught by at least one pin.

Sources: sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...",
section "Что именно изменилось" (fixed-size state; read the stored value for the
key, compare, write only the correction; one forgetting coefficient per state row
versus Gated DeltaNet's single one); m.lqnn.cn/news/205170, section
"KDA 与 Gated Attention：每 4 层只留 1 层全注意力" (kernel-4 causal conv with an
incremental cache; state = state * exp(gate) + delta, delta = residual * sigmoid(beta),
beta in (0, 1)).
"""
from __future__ import annotations

import numpy as np

import oracle

TOL = 1e-12


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} (scale {scale:.3e})"


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def random_inputs(seed, T, H, dk, dv, strong=False, h0=True):
    rng = np.random.default_rng(seed)
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    beta = _sigmoid(rng.standard_normal((T, H)))
    u = rng.normal(4.0, 1.0, (T, H, dk))
    if strong:
        u[..., : max(1, dk // 8)] = np.minimum(rng.normal(-1.0, 0.5, (T, H, max(1, dk // 8))),
                                               -0.05)
    g = np.log(_sigmoid(u))
    S0 = rng.normal(0.0, 0.3, (1, H, dk, dv)) if h0 else None
    return q, k, v, g, beta, S0


# --------------------------------------------------------------------------- #
# Delta rule: write / read                                                     #
# --------------------------------------------------------------------------- #

def pin_orthonormal_write_read(lib):
    """g=0, beta=1, orthonormal keys: S_m = (I - sum k_i k_i^T) S_0 + sum k_i v_i^T,
    so reading any written key returns its value exactly."""
    rng = np.random.default_rng(1)
    dk, dv, m = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :m].T                          # m orthonormal rows
    vals = rng.standard_normal((m, dv))
    S0 = rng.standard_normal((1, 1, dk, dv))
    q = _unit(rng.standard_normal((m, 1, dk)))
    o, S = oracle.kda_fwd(q, keys[:, None, :], vals[:, None, :], np.zeros((m, 1, dk)),
                          np.ones((m, 1)), 1.0, S0, lib=lib)
    proj = np.eye(dk) - keys.T @ keys
    expect = proj @ S0[0, 0] + keys.T @ vals
    _close(S[0, 0], expect, what="S_m closed form")
    _close(keys @ S[0, 0], vals, what="S^T k_i = v_i")


def pin_same_key_last_value_wins(lib):
    """beta=1, g=0: writing (k, v1) then (k, v2) leaves S^T k = v2."""
    rng = np.random.default_rng(2)
    dk, dv = 6, 4
    kk = _unit(rng.standard_normal(dk))
    v1, v2 = rng.standard_normal(dv), rng.standard_normal(dv)
    S0 = rng.standard_normal((1, 1, dk, dv))
    k = np.stack([kk, kk])[:, None, :]
    v = np.stack([v1, v2])[:, None, :]
    o, S = oracle.kda_fwd(k, k, v, np.zeros((2, 1, dk)), np.ones((2, 1)), 1.0, S0, lib=lib)
    _close(S[0, 0].T @ kk, v2, what="last value wins")
    _close(o[1, 0], v2, what="o_2 = S_2^T k = v2")


# --------------------------------------------------------------------------- #
# Decay                                                                        #
# --------------------------------------------------------------------------- #

def pin_beta_zero_pure_decay(lib):
    """beta=0: S_T = diag(exp(sum_t g_t)) S_0 and o_t = scale * S_0^T (exp(sum_{s<=t} g_s) * q_t)."""
    q, k, v, g, beta, S0 = random_inputs(3, 7, 2, 6, 5)
    g = g * 3.0  # wider range of per-row decays
    scale = 0.75
    o, S = oracle.kda_fwd(q, k, v, g, np.zeros_like(beta), scale, S0, lib=lib)
    cum = np.cumsum(g, axis=0)
    for h in range(2):
        _close(S[0, h], np.exp(cum[-1, h])[:, None] * S0[0, h], what="decayed state")
        for t in range(7):
            _close(o[t, h], scale * S0[0, h].T @ (np.exp(cum[t, h]) * q[t, h]),
                   what=f"decayed read t={t}")


# --------------------------------------------------------------------------- #
# Per-row gate vs the scalar gate of Gated DeltaNet                            #
# --------------------------------------------------------------------------- #

def pin_equal_gates_are_gated_deltanet(lib):
    """g_t = alpha_t * 1 makes KDA the scalar-gated DeltaNet (Householder form)."""
    q, k, v, g, beta, S0 = random_inputs(4, 9, 3, 8, 6)
    alpha = g[..., 0].copy()
    gg = np.repeat(alpha[..., None], 8, axis=-1)
    o1, S1 = oracle.kda_fwd(q, k, v, gg, beta, 1.0, S0, lib=lib)
    o2, S2 = oracle.gdn_fwd(q, k, v, alpha, beta, 1.0, S0, lib=lib)
    _close(o1, o2, what="o vs GDN")
    _close(S1, S2, what="S vs GDN")


# --------------------------------------------------------------------------- #
# Hand-unrolled closed forms                                                   #
# --------------------------------------------------------------------------- #

def pin_T1_closed_form(lib):
    q, k, v, g, beta, S0 = random_inputs(5, 1, 2, 7, 4)
    scale = 0.5
    o, S = oracle.kda_fwd(q, k, v, g, beta, scale, S0, lib=lib)
    for h in range(2):
        P = np.exp(g[0, h])[:, None] * S0[0, h]
        u = v[0, h] - P.T @ k[0, h]
        _close(S[0, h], P + beta[0, h] * np.outer(k[0, h], u), what="S_1")
        _close(o[0, h], scale * (P.T @ q[0, h] + beta[0, h] * (k[0, h] @ q[0, h]) * u),
               what="o_1")
    # zero initial state: o_1 = beta (k.q) v, S_1 = beta k v^T
    o, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, None, lib=lib)
    for h in range(2):
        _close(o[0, h], beta[0, h] * (k[0, h] @ q[0, h]) * v[0, h], what="o_1 zero state")
        _close(S[0, h], beta[0, h] * np.outer(k[0, h], v[0, h]), what="S_1 zero state")


def pin_T2_closed_form(lib):
    q, k, v, g, beta, S0 = random_inputs(6, 2, 2, 6, 5)
    o, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0, lib=lib)
    for h in range(2):
        D1, D2 = np.exp(g[0, h]), np.exp(g[1, h])
        P1 = D1[:, None] * S0[0, h]
        u1 = v[0, h] - P1.T @ k[0, h]
        k1, k2, q2 = k[0, h], k[1, h], q[1, h]
        b1, b2 = beta[0, h], beta[1, h]
        u2 = v[1, h] - P1.T @ (D2 * k2) - b1 * (k1 @ (D2 * k2)) * u1
        o2 = P1.T @ (D2 * q2) + b1 * (k1 @ (D2 * q2)) * u1 + b2 * (k2 @ q2) * u2
        S2 = D2[:, None] * P1 + b1 * np.outer(D2 * k1, u1) + b2 * np.outer(k2, u2)
        _close(o[1, h], o2, what="o_2")
        _close(S[0, h], S2, what="S_2")


# --------------------------------------------------------------------------- #
# Structure                                                                    #
# --------------------------------------------------------------------------- #

def pin_linearity(lib):
    """(o, S_T) is jointly linear in (V, S_0) for fixed q, k, g, beta."""
    q, k, v1, g, beta, S01 = random_inputs(7, 11, 2, 6, 5)
    rng = np.random.default_rng(70)
    v2 = rng.standard_normal(v1.shape)
    S02 = rng.standard_normal(S01.shape)
    a, b = 0.7, -1.3
    oa, Sa = oracle.kda_fwd(q, k, v1, g, beta, 1.0, S01, lib=lib)
    ob, Sb = oracle.kda_fwd(q, k, v2, g, beta, 1.0, S02, lib=lib)
    oc, Sc = oracle.kda_fwd(q, k, a * v1 + b * v2, g, beta, 1.0, a * S01 + b * S02, lib=lib)
    _close(oc, a * oa + b * ob, what="o linear")
    _close(Sc, a * Sa + b * Sb, what="S linear")


def pin_column_permutation(lib):
    """Permuting the value channels of V and S_0 permutes o and S_T the same way."""
    q, k, v, g, beta, S0 = random_inputs(8, 9, 2, 6, 7)
    perm = np.random.default_rng(80).permutation(7)
    o, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0, lib=lib)
    op, Sp = oracle.kda_fwd(q, k, v[..., perm], g, beta, 1.0, S0[..., perm], lib=lib)
    _close(op, o[..., perm], what="o permuted")
    _close(Sp, S[..., perm], what="S permuted")


def pin_varlen_equals_separate(lib):
    """Packed sequences give exactly what separate runs give."""
    lens = [3, 1, 6, 4]
    cu = np.cumsum([0] + lens)
    q, k, v, g, beta, _ = random_inputs(9, cu[-1], 2, 5, 4)
    rng = np.random.default_rng(90)
    h0 = rng.standard_normal((len(lens), 2, 5, 4))
    o, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, h0, cu, lib=lib)
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = oracle.kda_fwd(q[sl], k[sl], v[sl], g[sl], beta[sl], 1.0, h0[n:n + 1], lib=lib)
        assert np.array_equal(o[sl], on), "packed o differs from a separate run"
        assert np.array_equal(S[n], Sn[0]), "packed state differs from a separate run"


def pin_split_resume(lib):
    """run(T1) then run(T2, h0 = ht) equals run(T1 + T2)."""
    q, k, v, g, beta, S0 = random_inputs(10, 13, 2, 6, 5)
    o, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0, lib=lib)
    o1, S1 = oracle.kda_fwd(q[:5], k[:5], v[:5], g[:5], beta[:5], 1.0, S0, lib=lib)
    o2, S2 = oracle.kda_fwd(q[5:], k[5:], v[5:], g[5:], beta[5:], 1.0, S1, lib=lib)
    assert np.array_equal(np.concatenate([o1, o2]), o), "split outputs differ"
    assert np.array_equal(S2, S), "split final state differs"


def pin_contraction(lib):
    """g <= 0, |k| = 1, beta in (0,1): |S_t|_2 <= |S_{t-1}|_2 + beta_t |v_t| at every step,
    and strong (skewed) gates give finite results."""
    q, k, v, g, beta, S0 = random_inputs(11, 40, 2, 8, 6, strong=True)
    S = S0
    for t in range(40):
        o, Sn = oracle.kda_fwd(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1],
                               1.0, S, lib=lib)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(Sn))
        for h in range(2):
            lhs = np.linalg.norm(Sn[0, h], 2)
            rhs = np.linalg.norm(S[0, h], 2) + beta[t, h] * np.linalg.norm(v[t, h])
            assert lhs <= rhs * (1 + 1e-12), f"state grew beyond the contraction bound at t={t}"
        S = Sn


def pin_transition_affine(lib):
    """A stretch started from S ends in M S + (its end state from zero): checked against the
    recurrence itself from several starting states, over packed sequences of uneven length."""
    q, k, v, g, beta, _ = random_inputs(12, 23, 2, 6, 5, strong=True, h0=False)
    cu = np.array([0, 9, 9, 23])
    rng = np.random.default_rng(13)
    m = oracle.transition(k, g, beta, cu, lib=lib)
    _, S_zero = oracle.kda_fwd(q, k, v, g, beta, 1.0, None, cu, lib=lib)
    for _ in range(2):
        S0 = rng.normal(0.0, 1.0, (3, 2, 6, 5))
        _, S = oracle.kda_fwd(q, k, v, g, beta, 1.0, S0, cu, lib=lib)
        _close(S, np.einsum("nhij,nhjc->nhic", m, S0) + S_zero, tol=1e-12, what="affine in h0")
    _close(m[1], np.broadcast_to(np.eye(6), (2, 6, 6)), tol=0.0, what="empty sequence")


def pin_transition_closed_forms(lib):
    """beta = 0: M = diag(exp(sum_t g_t)). One token with g = 0: M = I - beta k k^T (M k =
    (1 - beta |k|^2) k, M x = x for x orthogonal to k). det M = exp(sum g) prod (1 - beta_t |k_t|^2)
    (the matrix determinant lemma). Two stretches compose as M(later) M(earlier)."""
    _, k, _, g, beta, _ = random_inputs(14, 7, 1, 5, 5, h0=False)
    m = oracle.transition(k, g, np.zeros_like(beta), lib=lib)
    _close(m[0, 0], np.diag(np.exp(g[:, 0].sum(axis=0))), tol=1e-14, what="beta = 0")
    kk = np.array([[[0.6, 0.0, -0.8, 0.0, 0.0]]])
    m1 = oracle.transition(kk, np.zeros_like(kk), np.array([[0.3]]), lib=lib)[0, 0]
    _close(m1 @ kk[0, 0], 0.7 * kk[0, 0], tol=1e-15, what="M k")
    x = np.array([0.8, 0.1, 0.6, -2.0, 0.5])
    _close(m1 @ x, x, tol=1e-15, what="M x, x orthogonal to k")
    m = oracle.transition(k, g, beta, lib=lib)[0, 0]
    det = np.exp(g[:, 0].sum()) * np.prod(1.0 - beta[:, 0] * np.sum(k[:, 0] ** 2, axis=-1))
    _close(np.linalg.det(m), det, tol=1e-12, what="determinant")
    ma = oracle.transition(k[:3], g[:3], beta[:3], lib=lib)[0, 0]
    mb = oracle.transition(k[3:], g[3:], beta[3:], lib=lib)[0, 0]
    _close(m, mb @ ma, tol=1e-13, what="composition order")


# --------------------------------------------------------------------------- #
# Conv prologue                                                                #
# --------------------------------------------------------------------------- #

def _torch_conv_silu(x, w):
    """torch CPU conv1d(groups=C, padding=K-1)[..., :T] followed by SiLU."""
    import torch
    xt = torch.from_numpy(np.ascontiguousarray(x.T))[None]        # [1, C, T]
    wt = torch.from_numpy(np.ascontiguousarray(w))[:, None, :]    # [C, 1, K]
    y = torch.nn.functional.conv1d(xt, wt, padding=w.shape[1] - 1, groups=w.shape[0])
    y = y[..., : x.shape[0]]
    return torch.nn.functional.silu(y)[0].T.numpy()


def pin_conv_matches_torch(lib):
    rng = np.random.default_rng(12)
    for K in (2, 4):
        x = rng.standard_normal((9, 6))
        w = rng.normal(0, 0.5, (6, K))
        y, cache = oracle.conv_silu(x, w, None, None, lib=lib)
        _close(y, _torch_conv_silu(x, w), tol=1e-12, what=f"conv K={K}")
        _close(cache[0], x[-(K - 1):].T, what="cache = last K-1 inputs")


def pin_conv_varlen_and_cache(lib):
    """The conv never crosses sequence boundaries; token-by-token calls with the cache
    reproduce the full-sequence conv (including sequences shorter than K-1)."""
    rng = np.random.default_rng(13)
    lens = [5, 2, 1, 7]
    cu = np.cumsum([0] + lens)
    C, K = 4, 4
    x = rng.standard_normal((cu[-1], C))
    w = rng.normal(0, 0.5, (C, K))
    y, cache = oracle.conv_silu(x, w, None, cu, lib=lib)
    for n in range(len(lens)):
        yn, cn = oracle.conv_silu(x[cu[n]:cu[n + 1]], w, None, None, lib=lib)
        assert np.array_equal(yn, y[cu[n]:cu[n + 1]])
        assert np.array_equal(cn[0], cache[n])
        ext = np.concatenate([np.zeros((K - 1, C)), x[cu[n]:cu[n + 1]]])
        _close(cache[n], ext[-(K - 1):].T, what="cache across the history boundary")
        # step mode: one token at a time, history carried in the cache
        st = np.zeros((1, C, K - 1))
        for t in range(lens[n]):
            ys, st = oracle.conv_silu(x[cu[n] + t:cu[n] + t + 1], w, st, None, lib=lib)
            _close(ys[0], y[cu[n] + t], what="step conv")
        _close(st[0], cache[n], what="step cache")


def pin_l2norm(lib):
    rng = np.random.default_rng(14)
    x = rng.standard_normal((5, 3, 16))
    eps = 1e-6
    y = oracle.l2norm(x, eps, lib=lib)
    _close(y, x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps), what="l2norm")
    _close(np.linalg.norm(oracle.l2norm(x, 0.0, lib=lib), axis=-1), np.ones((5, 3)),
           what="unit norm")


def pin_prologue_composition(lib):
    """prologue = conv+SiLU on each of q/k/v with its own slice of the cache, then L2 on q, k."""
    rng = np.random.default_rng(15)
    T, H, dk, dv = 6, 2, 4, 3
    qr, kr = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk))
    vr = rng.standard_normal((T, H, dv))
    wq, wk = rng.normal(0, .5, (H * dk, 4)), rng.normal(0, .5, (H * dk, 4))
    wv = rng.normal(0, .5, (H * dv, 4))
    cs = rng.standard_normal((1, H * (2 * dk + dv), 3))
    q, k, v, cso = oracle.prologue(qr, kr, vr, wq, wk, wv, cs, None, 1e-6, lib=lib)
    ext = lambda x, c: np.concatenate([c[0].T, x.reshape(T, -1)])          # noqa: E731
    for x, w, lo, hi, out, nrm in ((qr, wq, 0, 8, q, True), (kr, wk, 8, 16, k, True),
                                   (vr, wv, 16, 22, v, False)):
        e = ext(x, cs[:, lo:hi])
        y = _torch_conv_silu(e, w)[3:].reshape(out.shape)
        if nrm:
            y = y / np.sqrt(np.sum(y * y, axis=-1, keepdims=True) + 1e-6)
        _close(out, y, tol=1e-12, what="prologue part")
        _close(cso[0, lo:hi], e[-3:].T, what="prologue cache slice")


# --------------------------------------------------------------------------- #
# Gate activation and output norm                                             #
# --------------------------------------------------------------------------- #
# m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...": the gate comes from a_log_bias
# and dt_bias, and delta is the residual times sigmoid(beta). sarnas.ru, section "Отвергнутые
# решения": every norm except the QK norms is a gated RMSNorm. The formulas are readings (the
# pages give only the inputs); the pins below fix them against closed forms and torch's CPU
# routines.

def pin_gate_closed_form(lib):
    """x + dt_bias = 0 and A_log = 0 give g = -log 2; A_log = log 3 triples it; a very negative
    A_log switches the decay off (g -> 0); a large logit makes softplus the identity."""
    x = np.zeros((2, 3, 4))
    _close(oracle.gate(x, np.zeros(3), np.zeros(12), lib=lib), -np.log(2.0) * np.ones_like(x),
           tol=1e-15, what="gate at zero")
    g = oracle.gate(x, np.log([1.0, 3.0, 1e-30]), np.zeros(12), lib=lib)
    _close(g[:, 1], -3 * np.log(2.0) * np.ones((2, 4)), tol=1e-14, what="gate A_log scale")
    assert np.all(np.abs(g[:, 2]) < 1e-29), "gate with A_log -> -inf"
    big = oracle.gate(np.full((1, 1, 2), 40.0), np.zeros(1), np.array([0.0, 5.0]), lib=lib)
    _close(big[0, 0], [-40.0, -45.0], tol=1e-15, what="gate softplus linear branch")


def pin_gate_matches_torch(lib):
    """Random logits, per-head A_log and per-channel dt_bias against torch's fp64 softplus."""
    import torch
    rng = np.random.default_rng(41)
    T, H, dk = 9, 3, 8
    x = rng.normal(0.0, 3.0, (T, H, dk))
    A_log = rng.normal(0.0, 1.0, H)
    dt = rng.normal(0.0, 1.0, (H, dk))
    ref = -(torch.exp(torch.from_numpy(A_log))[None, :, None] *
            torch.nn.functional.softplus(torch.from_numpy(x) + torch.from_numpy(dt)[None]))
    g = oracle.gate(x, A_log, dt.reshape(-1), lib=lib)
    _close(g, ref.numpy(), tol=1e-13, what="gate vs torch softplus")
    assert np.all(g <= 0.0), "gate must be a decay (g <= 0)"


def pin_sigmoid(lib):
    """beta = sigmoid(b): 1/2 at 0, sigmoid(-b) = 1 - sigmoid(b), and torch's fp64 sigmoid."""
    import torch
    b = np.random.default_rng(43).normal(0.0, 4.0, 50)
    s = oracle.sigmoid(b, lib=lib)
    _close(oracle.sigmoid(np.zeros(1), lib=lib), [0.5], tol=1e-16, what="sigmoid(0)")
    _close(s + oracle.sigmoid(-b, lib=lib), np.ones_like(b), tol=1e-15, what="sigmoid symmetry")
    _close(s, torch.sigmoid(torch.from_numpy(b)).numpy(), tol=1e-15, what="sigmoid vs torch")


def pin_gated_rmsnorm(lib):
    """A constant row normalises to its sign; a large gate passes the plain RMSNorm (torch's
    rms_norm); a zero gate halves it; and the norm is scale-free."""
    import torch
    rng = np.random.default_rng(47)
    dv = 16
    w = rng.normal(1.0, 0.2, dv)
    o = np.full((1, dv), -2.5)
    y = oracle.gated_rmsnorm(o, np.full((1, dv), 60.0), w, eps=0.0, lib=lib)
    _close(y[0], -w, tol=1e-14, what="rmsnorm of a constant row")
    o = rng.normal(0.0, 3.0, (5, 2, dv))
    z = rng.normal(0.0, 2.0, (5, 2, dv))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (dv,), torch.from_numpy(w), 1e-6)
    _close(oracle.gated_rmsnorm(o, np.full_like(o, 60.0), w, 1e-6, lib=lib), ref.numpy(),
           tol=1e-13, what="rmsnorm vs torch")
    _close(oracle.gated_rmsnorm(o, np.zeros_like(o), w, 1e-6, lib=lib), 0.5 * ref.numpy(),
           tol=1e-13, what="gate sigmoid(0) = 1/2")
    gref = ref * torch.sigmoid(torch.from_numpy(z))
    _close(oracle.gated_rmsnorm(o, z, w, 1e-6, lib=lib), gref.numpy(), tol=1e-13,
           what="gated rmsnorm vs torch")
    _close(oracle.gated_rmsnorm(7.0 * o, z, w, 0.0, lib=lib), oracle.gated_rmsnorm(o, z, w, 0.0, lib=lib),
           tol=1e-13, what="scale invariance")


ALL_PINS = [
    pin_orthonormal_write_read, pin_same_key_last_value_wins, pin_beta_zero_pure_decay,
    pin_equal_gates_are_gated_deltanet, pin_T1_closed_form, pin_T2_closed_form, pin_linearity,
    pin_column_permutation, pin_varlen_equals_separate, pin_split_resume, pin_contraction,
    pin_transition_affine, pin_transition_closed_forms,
    pin_conv_matches_torch, pin_conv_varlen_and_cache, pin_l2norm, pin_prologue_composition,
    pin_gate_closed_form, pin_gate_matches_torch, pin_sigmoid, pin_gated_rmsnorm,
]
