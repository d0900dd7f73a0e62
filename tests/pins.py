"""Pins of the fp64 oracle: checks against what the method's pages fix.

Each ``pin_*`` takes a loaded :class:`oracle.Oracle` and raises AssertionError
on a mismatch, so the same checks run on the real oracle
(``test_oracle_pins.py``) and on deliberately broken copies of it
(``test_oracle_mutants.py``).  Sources, by page and section:

  [DPR1]  "Complex KDA" review, section "Diagonal-plus-rank-one (DPR1) transition"
  [HH]    same page, "Delta rule and Householder reflection" (beta = 0, 1, 2)
  [STEPS] same page, "Method steps" (step 1 ranges, 2 the 2-D construction,
          3 Prop. 2, 4 group constructions)
  [CORE]  same page, "Core method" (commutator, discriminant, Theorem 8)
  [THM1]  same page, Theorem 1 / Figure 3 (orthogonal DPR1 matrices, ||A||_2 <= 1)
  [LA]    CyFA blog, section 2.1 (linear attention S_t = S_{t-1} + k v^T)
  [DR]    CyFA blog, section 2.2 (delta rule S_t = S_{t-1} + k (v - S^T k)^T)
  [CHUNK] CyFA blog, section 5.5 (chunk = 1 and chunk = 64 must agree)
  [FIG6]  "Complex KDA" review, "Experimental results", Figure 6 (the gate range or the
          strength range widened alone)
  [FIG5]  same page, Figure 5 (the kernels are measured forward plus backward; the pages give
          no backward formulas, so the backward oracle is pinned by calculus alone: finite
          differences, Euler identities of the linear arguments, closed forms)
  [DP2]   same page, "Research motivation" and "Experimental results" (5): DeltaProduct2 reaches
          plane rotations with two rank-one delta-rule updates per token (one more key and
          value), the composition of two Householder reflections
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from chunkwise_ref import chunk_fwd_one

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
INF = float("inf")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _unit(rng, *shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rel(x, ref):
    n = np.linalg.norm(ref)
    return np.linalg.norm(x - ref) / (n if n > 0 else 1.0)


def _one(orc, q, k, v, alpha, beta, S0, signed_gate=2):
    """Oracle forward on one sequence and head given [T,d] arrays."""
    T, dk = q.shape
    dv = v.shape[1]
    o, S = orc.ckda_fwd(q.reshape(1, T, 1, dk), k.reshape(1, T, 1, dk), v.reshape(1, T, 1, dv),
                        alpha.reshape(1, T, 1, dk), np.asarray(beta, float).reshape(1, T, 1),
                        None if S0 is None else S0.reshape(1, 1, dk, dv),
                        signed_gate=signed_gate, threads=1)
    return o.reshape(T, dv), S.reshape(dk, dv)


def _rot(x):
    return np.array([[math.cos(x), -math.sin(x)], [math.sin(x), math.cos(x)]])


# ---------------------------------------------------------------- activation


def pin_gate_activation(orc):
    """[STEPS] step 1: CKDA alpha = 2 sigma(a) - 1 = tanh(a/2), beta = 2 sigma(b) = 1 + tanh(b/2);
    KDA alpha = sigma(a) = (1 + tanh(a/2)) / 2.  Exact endpoints at +-inf."""
    a = np.array([-INF, -30.0, -3.0, -0.7, 0.0, 1e-9, 0.7, 3.0, 30.0, INF])
    al1, be1 = orc.gates(a, a, 1)
    al0, be0 = orc.gates(a, a, 0)
    al2, be2 = orc.gates(a, a, 2)
    th = np.tanh(a / 2)
    assert np.allclose(al1, th, rtol=1e-13, atol=1e-15)
    assert np.allclose(be1, 1 + th, rtol=1e-13, atol=1e-15)
    assert np.allclose(al0, (1 + th) / 2, rtol=1e-13, atol=1e-15)
    assert np.allclose(be0, (1 + th) / 2, rtol=1e-13, atol=1e-15)
    assert al1[0] == -1.0 and al1[-1] == 1.0 and al1[4] == 0.0
    assert be1[0] == 0.0 and be1[-1] == 2.0 and be1[4] == 1.0
    assert al0[0] == 0.0 and al0[-1] == 1.0 and al0[4] == 0.5
    assert np.array_equal(al2, a) and np.array_equal(be2, a)


def pin_single_range_variants(orc):
    """[FIG6]: signed_gate 3 widens the gate range alone (alpha = 2 sigma(a) - 1 = tanh(a/2),
    beta = sigma(b)), 4 the strength range alone (alpha = sigma(a), beta = 2 sigma(b)).  The
    gates against tanh closed forms, and a whole forward in each form against the raw form
    fed with those closed forms."""
    a = np.array([-INF, -30.0, -3.0, -0.7, 0.0, 1e-9, 0.7, 3.0, 30.0, INF])
    th = np.tanh(a / 2)
    al3, be3 = orc.gates(a, a, 3)
    al4, be4 = orc.gates(a, a, 4)
    assert np.allclose(al3, th, rtol=1e-13, atol=1e-15)
    assert np.allclose(be3, (1 + th) / 2, rtol=1e-13, atol=1e-15)
    assert np.allclose(al4, (1 + th) / 2, rtol=1e-13, atol=1e-15)
    assert np.allclose(be4, 1 + th, rtol=1e-13, atol=1e-15)
    assert al3[0] == -1.0 and al3[-1] == 1.0 and be3[0] == 0.0 and be3[-1] == 1.0
    assert al4[0] == 0.0 and al4[-1] == 1.0 and be4[0] == 0.0 and be4[-1] == 2.0
    rng = np.random.default_rng(61)
    T, dk, dv = 23, 5, 3
    q, k, v = _unit(rng, T, dk), _unit(rng, T, dk), rng.standard_normal((T, dv))
    la, lb = rng.standard_normal((T, dk)) * 2, rng.standard_normal(T) * 2
    S0 = rng.standard_normal((dk, dv))
    sig = lambda x: (1 + np.tanh(x / 2)) / 2
    for sg, alpha, beta in ((3, np.tanh(la / 2), sig(lb)), (4, sig(la), 1 + np.tanh(lb / 2))):
        o, S = _one(orc, q, k, v, la, lb, S0, signed_gate=sg)
        ro, rS = _one(orc, q, k, v, alpha, beta, S0, signed_gate=2)
        assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12, sg


# ------------------------------------------------------- closed-form cases


def pin_beta_zero(orc):
    """(i) [HH] beta = 0: no write, S_T = Diag(prod alpha) S0, o_t = (Diag(G_t) S0)^T q_t."""
    rng = np.random.default_rng(1)
    T, dk, dv = 9, 5, 4
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(-1, 1, (T, dk))
    S0 = rng.standard_normal((dk, dv))
    o, S = _one(orc, q, k, v, alpha, np.zeros(T), S0)
    G = np.cumprod(alpha, axis=0)
    assert _rel(S, G[-1][:, None] * S0) < 1e-14
    for t in range(T):
        assert _rel(o[t], (G[t][:, None] * S0).T @ q[t]) < 1e-14
    # the same through the logits: b = -inf gives beta = 0 exactly in both forms
    for sg in (0, 1):
        a = rng.standard_normal((T, dk))
        al, _ = orc.gates(a, np.zeros(1), sg)
        o2, S2 = _one(orc, q, k, v, a, np.full(T, -INF), S0, signed_gate=sg)
        G2 = np.cumprod(al, axis=0)
        assert _rel(S2, G2[-1][:, None] * S0) < 1e-14


def pin_frozen_state(orc):
    """(ii) [HH] alpha = 1, beta = 0: identity transition, S_t = S_0, o_t = S_0^T q_t.
    Driven through KDA logits a = +inf (alpha = 1) and b = -inf (beta = 0)."""
    rng = np.random.default_rng(2)
    T, dk, dv = 7, 6, 3
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    v = rng.standard_normal((T, dv))
    S0 = rng.standard_normal((dk, dv))
    o, S = _one(orc, q, k, v, np.full((T, dk), INF), np.full(T, -INF), S0, signed_gate=0)
    assert np.array_equal(S, S0)
    assert _rel(o, q @ S0) < 1e-15


def pin_linear_attention(orc):
    """(iii) [LA] alpha = 1, beta = 1, orthonormal keys, S0 = 0: the erase term vanishes and
    S_t = sum_{j<=t} k_j v_j^T, o_t = sum_{j<=t} (k_j . q_t) v_j."""
    rng = np.random.default_rng(3)
    dk, dv, T = 8, 5, 8
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T]                              # orthonormal rows
    q, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    o, S = _one(orc, q, k, v, np.ones((T, dk)), np.ones(T), None)
    for t in range(T):
        St = sum(np.outer(k[j], v[j]) for j in range(t + 1))
        assert _rel(o[t], sum((k[j] @ q[t]) * v[j] for j in range(t + 1))) < 1e-12
    assert _rel(S, St) < 1e-12


def pin_delta_rule(orc):
    """(iv) [DR] alpha = 1, beta = 1 is the textbook delta rule S + k (v - S^T k)^T."""
    rng = np.random.default_rng(4)
    T, dk, dv = 12, 6, 4
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    v = rng.standard_normal((T, dv))
    S0 = rng.standard_normal((dk, dv))
    o, S = _one(orc, q, k, v, np.ones((T, dk)), np.ones(T), S0)
    R = S0.copy()
    for t in range(T):
        R = R + np.outer(k[t], v[t] - R.T @ k[t])
        assert _rel(o[t], R.T @ q[t]) < 1e-13
    assert _rel(S, R) < 1e-13


def pin_transition_beta_012(orc):
    """(v) [HH] unit k, alpha = 1: beta = 0 identity, 1 projection, 2 Householder reflection."""
    rng = np.random.default_rng(5)
    n = 7
    k = _unit(rng, n)
    ones = np.ones(n)
    I = np.eye(n)
    A0 = orc.transition(k, ones, 0.0)
    A1 = orc.transition(k, ones, 1.0)
    A2 = orc.transition(k, ones, 2.0)
    assert np.allclose(A0, I, atol=1e-15)
    assert np.allclose(A1 @ A1, A1, atol=1e-14) and np.allclose(A1 @ k, 0, atol=1e-14)
    assert np.allclose(A1, A1.T, atol=1e-15)
    x = rng.standard_normal(n)
    x -= (x @ k) * k                          # orthogonal to k: kept by the projector
    assert np.allclose(A1 @ x, x, atol=1e-14)
    assert np.allclose(A2 @ A2, I, atol=1e-14) and np.allclose(A2.T @ A2, I, atol=1e-14)
    assert np.allclose(A2 @ k, -k, atol=1e-14) and np.allclose(A2 @ x, x, atol=1e-14)


def pin_commutator(orc):
    """(vi) [CORE] (H_k D - D H_k)_ij = beta k_i k_j (alpha_i - alpha_j), H_k = I - beta k k^T;
    the transition is H_k D (gate applied first); a scalar gate commutes."""
    rng = np.random.default_rng(6)
    n = 6
    for _ in range(5):
        k = _unit(rng, n)
        alpha = rng.uniform(-1, 1, n)
        beta = rng.uniform(0, 2)
        HD = orc.transition(k, alpha, beta)
        H = orc.transition(k, np.ones(n), beta)
        D = orc.transition(k, alpha, 0.0)
        assert np.allclose(D, np.diag(alpha), atol=1e-15)
        assert np.allclose(HD, H @ D, atol=1e-14)
        expect = beta * np.outer(k, k) * (alpha[:, None] - alpha[None, :])
        assert np.allclose(HD - D @ H, expect, atol=1e-14)
        c = rng.uniform(-1, 1)
        Hs = orc.transition(k, np.full(n, c), beta)
        assert np.allclose(Hs, c * H, atol=1e-15)       # scalar gate: H D = D H


def pin_spectrum_2d(orc):
    """(vii) [CORE], [STEPS] step 3: trace, determinant and complex pair of the 2-D transition,
    on the golden cases and on a grid."""
    g = _golden("spectrum_2d.json")
    for c in g["cases"]:
        t = c["theta"]
        A = orc.transition([math.cos(t), math.sin(t)], c["alpha"], c["beta"])
        assert abs(np.trace(A) - c["trace"]) < 1e-14
        assert abs(np.linalg.det(A) - c["det"]) < 1e-14
        lam = np.linalg.eigvals(A)
        lam = lam[np.argsort(-lam.imag)]
        assert abs(lam[0].real - c["re"]) < 1e-13 and abs(lam[0].imag - c["im"]) < 1e-13
    for al in np.linspace(-0.95, 0.95, 9):
        for t in np.linspace(0.05, 3.0, 11):
            A = orc.transition([math.cos(t), math.sin(t)], [al, 1.0], 2.0)
            disc = (1 - al) ** 2 * math.cos(2 * t) ** 2 + 4 * al
            lam = np.linalg.eigvals(A)
            if disc < -1e-9:
                assert np.all(np.abs(lam.imag) > 1e-9)
                assert np.allclose(np.abs(lam), math.sqrt(-al), atol=1e-12)
            elif disc > 1e-9:
                assert np.all(np.abs(lam.imag) < 1e-12)
    for be in np.linspace(0.1, 1.9, 10):
        for t in np.linspace(0.05, 3.0, 11):
            A = orc.transition([math.cos(t), math.sin(t)], [-1.0, 1.0], be)
            assert abs(np.trace(A) - be * math.cos(2 * t)) < 1e-14
            assert abs(np.linalg.det(A) - (be - 1)) < 1e-14
            lam = np.linalg.eigvals(A)
            crit = be ** 2 * math.cos(2 * t) ** 2 - 4 * (be - 1)
            if crit < -1e-9:
                assert np.allclose(np.abs(lam), math.sqrt(be - 1), atol=1e-12)
            elif crit > 1e-9:
                assert np.all(np.abs(lam.imag) < 1e-12)


def pin_exact_rotation(orc):
    """(viii) [STEPS] steps 2 and 4: CKDA logits a = (-inf, +inf), b = +inf give alpha = (-1, 1),
    beta = 2 exactly; with k = (cos t, sin t), v = 0, S0 = I one token is R(2t), and tokens
    x_t with t = pi x_t / m multiply to R(2 pi sum x / m) (addition mod m)."""
    g = _golden("rotation_2d.json")
    for c in g["cases"]:
        thetas = c["thetas"] if c["m"] == 0 else [math.pi * x / c["m"] for x in c["tokens"]]
        T = len(thetas)
        k = np.array([[math.cos(t), math.sin(t)] for t in thetas])
        a = np.tile([-INF, INF], (T, 1))
        q = np.tile([1.0, 0.0], (T, 1))
        o, S = _one(orc, q, k, np.zeros((T, 2)), a, np.full(T, INF), np.eye(2), signed_gate=1)
        assert np.allclose(S, np.array(c["expect"]), atol=1e-14)
        assert np.allclose(o[-1], S.T @ q[-1], atol=1e-15)
    rng = np.random.default_rng(8)
    for m in (3, 5, 7):
        x = rng.integers(0, m, size=40)
        k = np.stack([np.cos(np.pi * x / m), np.sin(np.pi * x / m)], axis=1)
        a = np.tile([-INF, INF], (len(x), 1))
        _, S = _one(orc, np.zeros((len(x), 2)), k, np.zeros((len(x), 2)), a,
                    np.full(len(x), INF), np.eye(2), signed_gate=1)
        assert np.allclose(S, _rot(2 * np.pi * (x.sum() % m) / m), atol=1e-12)


def pin_non_expansive(orc):
    """(ix) [THM1] ||A||_2 <= 1 for alpha in [-1,1]^n, beta in [0,2], ||k|| = 1."""
    rng = np.random.default_rng(9)
    worst = 0.0
    for _ in range(300):
        n = int(rng.integers(2, 12))
        A = orc.transition(_unit(rng, n), rng.uniform(-1, 1, n), rng.uniform(0, 2))
        worst = max(worst, np.linalg.norm(A, 2))
    assert worst <= 1 + 1e-12
    # outside the range (beta > 2) the bound fails, so the check is not vacuous
    k = _unit(rng, 4)
    assert np.linalg.norm(orc.transition(k, np.ones(4), 2.5), 2) > 1.4


def pin_orthogonal_case(orc):
    """(x) [THM1] alpha in {+-1}^n, beta = 2: A^T A = I; with v = 0 the recurrence keeps ||S||_F."""
    rng = np.random.default_rng(10)
    n = 6
    for _ in range(10):
        A = orc.transition(_unit(rng, n), rng.choice([-1.0, 1.0], n), 2.0)
        assert np.allclose(A.T @ A, np.eye(n), atol=1e-14)
    T, dv = 1000, 3
    k = _unit(rng, T, n)
    a = rng.choice([-INF, INF], (T, n))
    S0 = rng.standard_normal((n, dv))
    _, S = _one(orc, np.zeros((T, n)), k, np.zeros((T, dv)), a, np.full(T, INF), S0, 1)
    assert abs(np.linalg.norm(S) - np.linalg.norm(S0)) < 1e-11 * np.linalg.norm(S0)


def pin_one_complex_pair(orc):
    """(xi) [CORE] Theorem 8: at most one non-real conjugate pair per transition, and none
    unless beta > 1 and some gate is negative."""
    rng = np.random.default_rng(11)
    seen_pair = False
    for _ in range(400):
        n = int(rng.integers(2, 16))
        alpha = rng.uniform(-1, 1, n)
        beta = rng.uniform(0, 2)
        lam = np.linalg.eigvals(orc.transition(_unit(rng, n), alpha, beta))
        nonreal = int(np.sum(np.abs(lam.imag) > 1e-9))
        assert nonreal <= 2
        if nonreal:
            seen_pair = True
            assert beta > 1 and alpha.min() < 0
        lam_pos = np.linalg.eigvals(orc.transition(_unit(rng, n), np.abs(alpha), beta))
        assert np.all(np.abs(lam_pos.imag) < 1e-9)            # KDA range: real spectrum
    assert seen_pair


def pin_sign_gauge(orc):
    """(xii) [STEPS] step 5: the cumulative gate sign s_t = prod_{tau<=t} sign(alpha_tau) moves
    into the keys and queries.  CKDA(q, k, v, alpha, beta, S0) equals the non-negative-gate
    recurrence on (s*q, s*k, v, |alpha|, beta, S0), with S_T = Diag(s_T) S~_T."""
    rng = np.random.default_rng(12)
    T, dk, dv = 40, 7, 5
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(-1, 1, (T, dk))
    alpha[5, 2] = 0.0
    beta = rng.uniform(0, 2, T)
    S0 = rng.standard_normal((dk, dv))
    o, S = _one(orc, q, k, v, alpha, beta, S0)
    s = np.cumprod(np.where(alpha < 0, -1.0, 1.0), axis=0)
    o2, S2 = _one(orc, s * q, s * k, v, np.abs(alpha), beta, S0)
    assert _rel(o2, o) < 1e-12
    assert _rel(s[-1][:, None] * S2, S) < 1e-12


def pin_explicit_products(orc):
    """(xiii) [DPR1] the rank-one update equals the dense product S_T = A_T ... A_1 S0 (v = 0)
    and the explicit-matrix recurrence for general v."""
    rng = np.random.default_rng(13)
    T, dk, dv = 15, 5, 3
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    alpha = rng.uniform(-1, 1, (T, dk))
    beta = rng.uniform(0, 2, T)
    S0 = rng.standard_normal((dk, dv))
    _, S = _one(orc, q, k, np.zeros((T, dv)), alpha, beta, S0)
    M = np.eye(dk)
    for t in range(T):
        M = orc.transition(k[t], alpha[t], beta[t]) @ M
    assert _rel(S, M @ S0) < 1e-13
    v = rng.standard_normal((T, dv))
    o1, S1 = _one(orc, q, k, v, alpha, beta, S0)
    o2, S2 = orc.ckda_fwd_explicit(q, k, v, alpha, beta, S0, signed_gate=2)
    assert _rel(o1, o2) < 1e-13 and _rel(S1, S2) < 1e-13


def pin_chunkwise_equals_sequential(orc):
    """(xiv) [CHUNK], [DPR1] WY chunk-wise form: an independent numpy UT-transform forward
    agrees with the sequential oracle for chunk sizes 1, 2, 4, 16 and 64, with zero gates,
    +-1 gates and a ragged last chunk."""
    rng = np.random.default_rng(14)
    T, dk, dv = 83, 8, 6
    q, k = rng.standard_normal((T, dk)), _unit(rng, T, dk)
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(-1, 1, (T, dk))
    alpha[10, :3] = 0.0
    alpha[20:24, 4] = -1.0
    alpha[30, :] = 1.0
    beta = rng.uniform(0, 2, T)
    S0 = rng.standard_normal((dk, dv))
    o, S = _one(orc, q, k, v, alpha, beta, S0)
    for C in (1, 2, 4, 16, 64):
        oc, Sc = chunk_fwd_one(q, k, v, alpha, beta, S0, C)
        assert _rel(oc, o) < 1e-12, C
        assert _rel(Sc, S) < 1e-12, C


def pin_scalar_case(orc):
    """(xv) [DPR1] dk = dv = 1: hand-computed steps (golden file, exact rationals)."""
    g = _golden("scalar_two_steps.json")
    T = len(g["alpha"])
    col = lambda x: np.asarray(x, float).reshape(T, 1)
    o, S = _one(orc, col(g["q"]), col(g["k"]), col(g["v"]), col(g["alpha"]),
                np.asarray(g["beta"]), np.array([[g["S0"]]]), signed_gate=g["signed_gate"])
    assert np.allclose(o.ravel(), g["expect_o"], rtol=0, atol=1e-15)
    assert abs(S[0, 0] - g["expect_S_T"]) < 1e-15


def pin_split_resume(orc):
    """(xvi) the state is the whole summary: run(T1) then run(T2) from its S_T equals run(T1+T2);
    decode steps after a prefill equal a longer prefill; varlen packing equals separate runs."""
    rng = np.random.default_rng(16)
    T, H, dk, dv = 50, 3, 6, 5
    q = rng.standard_normal((1, T, H, dk))
    k = _unit(rng, 1, T, H, dk)
    v = rng.standard_normal((1, T, H, dv))
    a = rng.standard_normal((1, T, H, dk)) * 2
    b = rng.standard_normal((1, T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = orc.ckda_fwd(q, k, v, a, b, S0, signed_gate=1, threads=2)
    for T1 in (1, 17, 32):
        o1, S1 = orc.ckda_fwd(q[:, :T1], k[:, :T1], v[:, :T1], a[:, :T1], b[:, :T1], S0,
                              signed_gate=1)
        o2, S2 = orc.ckda_fwd(q[:, T1:], k[:, T1:], v[:, T1:], a[:, T1:], b[:, T1:], S1,
                              signed_gate=1)
        assert _rel(np.concatenate([o1, o2], axis=1), o) < 1e-13
        assert _rel(S2, S) < 1e-13
    # decode: the last 5 tokens one at a time
    T1 = T - 5
    _, St = orc.ckda_fwd(q[:, :T1], k[:, :T1], v[:, :T1], a[:, :T1], b[:, :T1], S0, signed_gate=1)
    St = St[0]
    for t in range(T1, T):
        od, St = orc.decode_step(q[:, t], k[:, t], v[:, t], a[:, t], b[:, t], St[None], 1)
        St = St[0]
        assert _rel(od[0], o[0, t]) < 1e-13
    assert _rel(St, S[0]) < 1e-13
    # varlen: three packed sequences (one empty) equal three separate calls
    cu = np.array([0, 20, 20, T], dtype=np.int32)
    S0v = rng.standard_normal((3, H, dk, dv))
    ov, Sv = orc.ckda_fwd(q, k, v, a, b, S0v, cu_seqlens=cu, signed_gate=1)
    for n in range(3):
        t0, t1 = cu[n], cu[n + 1]
        on, Sn = orc.ckda_fwd(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1], a[:, t0:t1], b[:, t0:t1],
                              S0v[n:n + 1], signed_gate=1)
        assert _rel(ov[:, t0:t1], on) < 1e-15 if t1 > t0 else True
        assert _rel(Sv[n], Sn[0]) < 1e-15
    assert np.array_equal(Sv[1], S0v[1])                 # empty sequence keeps S0


def pin_period_two(orc):
    """(xvii) [HH] adversarial UT case: every key equal and unit, beta = 2, alpha = 1 makes each
    transition the same reflection H (H k = -k), so with a constant v the state has period 2:
    S_2 = H(H S_0 + 2 k v^T) + 2 k v^T = S_0."""
    rng = np.random.default_rng(17)
    n, dv, T = 5, 4, 64
    k = np.tile(_unit(rng, n), (T, 1))
    v = np.tile(rng.standard_normal(dv), (T, 1))
    S0 = rng.standard_normal((n, dv))
    a = np.full((T, n), INF)
    _, S = _one(orc, np.zeros((T, n)), k, v, a, np.full(T, INF), S0, signed_gate=1)
    assert _rel(S, S0) < 1e-13
    _, S1 = _one(orc, np.zeros((T - 1, n)), k[:-1], v[:-1], a[:-1], np.full(T - 1, INF), S0, 1)
    assert _rel(S1, orc.transition(k[0], np.ones(n), 2.0) @ S0 + 2 * np.outer(k[0], v[0])) < 1e-13


# ---------------------------------------------------------------- backward ([FIG5])


def _bwd_case(rng, B, T, H, dk, dv, n_seqs=None):
    q = rng.standard_normal((B, T, H, dk))
    k = _unit(rng, B, T, H, dk)
    v = rng.standard_normal((B, T, H, dv))
    a = rng.standard_normal((B, T, H, dk)) * 1.5
    b = rng.standard_normal((B, T, H))
    N = B if n_seqs is None else n_seqs
    S0 = rng.standard_normal((N, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dS_T = rng.standard_normal((N, H, dk, dv))
    return [q, k, v, a, b, S0], dO, dS_T


def _check_fd(orc, args, dO, dS_T, sg, cu=None, h=1e-5, tol=1e-7):
    """Central differences of L = sum dO . o + sum dS_T . S_T in every input element."""
    def loss(xs):
        o, S = orc.ckda_fwd(*xs, cu_seqlens=cu, signed_gate=sg, threads=1)
        return float((dO * o).sum() + (dS_T * S).sum())

    grads = orc.ckda_bwd(*args, dO=dO, dS_T=dS_T, cu_seqlens=cu, signed_gate=sg, threads=1)
    for idx, (x, g) in enumerate(zip(args, grads)):
        fd = np.empty_like(x)
        for e in range(x.size):
            xs = list(args)
            xp, xm = x.copy(), x.copy()
            xp.flat[e] += h
            xm.flat[e] -= h
            xs[idx] = xp
            lp = loss(xs)
            xs[idx] = xm
            fd.flat[e] = (lp - loss(xs)) / (2 * h)
        assert _rel(g, fd) < tol, ("q k v a b S0".split()[idx], sg, _rel(g, fd))


def pin_bwd_finite_differences(orc):
    """[FIG5] every gradient of the backward oracle equals central finite differences of the
    forward, in all five gate forms; and across state checkpoints (sequences longer than 64
    tokens) with packed sequences, one of them empty."""
    rng = np.random.default_rng(70)
    args, dO, dS_T = _bwd_case(rng, 2, 11, 2, 3, 4)
    for sg in range(5):
        _check_fd(orc, args, dO, dS_T, sg)
    cu = np.array([0, 70, 70, 150], dtype=np.int32)
    args, dO, dS_T = _bwd_case(rng, 1, 150, 1, 2, 3, n_seqs=3)
    _check_fd(orc, args, dO, dS_T, 1, cu=cu)


def pin_bwd_euler_identities(orc):
    """[FIG5] exact identities of the linear arguments (Euler's theorem for functions of degree
    one): o is linear in q and S_T does not depend on q, so sum dq . q = sum dO . o; o and S_T
    are jointly linear in (v, S0), so sum dv . v + sum dS0 . S0 = L."""
    rng = np.random.default_rng(71)
    for sg in (0, 1):
        args, dO, dS_T = _bwd_case(rng, 2, 150, 2, 8, 6)
        q, k, v, a, b, S0 = args
        o, S = orc.ckda_fwd(*args, signed_gate=sg, threads=2)
        L = (dO * o).sum() + (dS_T * S).sum()
        dq, dk, dv, da, db, dS0 = orc.ckda_bwd(*args, dO=dO, dS_T=dS_T, signed_gate=sg, threads=2)
        assert abs((dq * q).sum() - (dO * o).sum()) < 1e-12 * np.abs(dO * o).sum()
        assert abs((dv * v).sum() + (dS0 * S0).sum() - L) < 1e-12 * (np.abs(dO * o).sum()
                                                                       + np.abs(dS_T * S).sum())


def pin_bwd_beta_zero(orc):
    """[FIG5] with beta = 0 the state is Diag(G_t) S0: closed forms of every gradient, the
    strength's taken through the write and erase terms it switches on
    (d S_s / d beta_t = Diag(g(s,t)) k_t (v_t - p_t)^T, p_t = S0^T Diag(G_t) k_t)."""
    rng = np.random.default_rng(72)
    T, dk, dv = 9, 4, 3
    q, k, v = rng.standard_normal((T, dk)), _unit(rng, T, dk), rng.standard_normal((T, dv))
    alpha = rng.uniform(-1, 1, (T, dk))
    S0, dO, dS_T = (rng.standard_normal(s) for s in ((dk, dv), (T, dv), (dk, dv)))
    r = lambda x, *s: x.reshape(*s)
    dq, dk_, dv_, da, db, dS0 = orc.ckda_bwd(r(q, 1, T, 1, dk), r(k, 1, T, 1, dk), r(v, 1, T, 1, dv),
                                             r(alpha, 1, T, 1, dk), np.zeros((1, T, 1)),
                                             r(S0, 1, 1, dk, dv), dO=r(dO, 1, T, 1, dv),
                                             dS_T=r(dS_T, 1, 1, dk, dv), signed_gate=2, threads=1)
    dq, dk_, dv_, da, db, dS0 = (x.reshape(-1, x.shape[-1]) if x.ndim == 4 else x
                                 for x in (dq, dk_, dv_, da, db, dS0))
    db = db.ravel()
    dS0 = dS0.reshape(dk, dv)

    def g(s, t):                       # prod_{r=t+1..s} alpha_r (1 when s == t)
        out = np.ones(dk)
        for x in range(t + 1, s + 1):
            out = out * alpha[x]
        return out

    def g_skip(s, t):                  # prod_{r<=s, r != t} alpha_r
        out = np.ones(dk)
        for x in range(s + 1):
            if x != t:
                out = out * alpha[x]
        return out

    G = [g(t, -1) for t in range(T)]
    assert np.abs(dk_).max() == 0.0 and np.abs(dv_).max() == 0.0
    for t in range(T):
        assert _rel(dq[t], (G[t][:, None] * S0) @ dO[t]) < 1e-13
    want = sum(np.outer(G[t] * q[t], dO[t]) for t in range(T)) + G[T - 1][:, None] * dS_T
    assert _rel(dS0, want) < 1e-13
    for t in range(T):
        want_a = sum(g_skip(s, t) * q[s] * (S0 @ dO[s]) for s in range(t, T))
        want_a = want_a + g_skip(T - 1, t) * (S0 * dS_T).sum(axis=1)
        assert _rel(da[t], want_a) < 1e-12
        dS_t = sum(np.outer(g(s, t) * q[s], dO[s]) for s in range(t, T)) + g(T - 1, t)[:, None] * dS_T
        p_t = S0.T @ (G[t] * k[t])
        assert abs(db[t] - (dS_t.T @ k[t]) @ (v[t] - p_t)) < 1e-12 * (1 + abs(db[t]))


def pin_bwd_linear_attention(orc):
    """[FIG5] [LA] alpha = 1, beta = 1, orthonormal keys, S0 = 0 (linear attention): the
    transitions are commuting projectors, so dv_j = sum_{t>=j} (k_j . q_t) dO_t + dS_T^T k_j,
    dq_t = sum_{j<=t} k_j (v_j . dO_t), dS0 = sum_t P_t q_t dO_t^T + P_T dS_T with
    P_t = I - sum_{j<=t} k_j k_j^T, dbeta_t = sum_{s>=t} (q_s . k_t)(v_t . dO_s) + k_t^T dS_T v_t,
    and dalpha_t,i = sum_{s>=t} (M_ts q_s)_i (S_{t-1} dO_s)_i + sum_j (M_tT dS_T)_ij (S_{t-1})_ij
    with M_ts = I - sum_{r=t..s} k_r k_r^T."""
    rng = np.random.default_rng(73)
    dk, dv, T = 8, 5, 7
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T]
    q, v, dO = rng.standard_normal((T, dk)), rng.standard_normal((T, dv)), rng.standard_normal((T, dv))
    dS_T = rng.standard_normal((dk, dv))
    r = lambda x, *s: x.reshape(*s)
    dq, _, dv_, da, db, dS0 = orc.ckda_bwd(r(q, 1, T, 1, dk), r(k, 1, T, 1, dk), r(v, 1, T, 1, dv),
                                           np.ones((1, T, 1, dk)), np.ones((1, T, 1)), None,
                                           dO=r(dO, 1, T, 1, dv), dS_T=r(dS_T, 1, 1, dk, dv),
                                           signed_gate=2, threads=1)
    dq, dv_, da = dq.reshape(T, dk), dv_.reshape(T, dv), da.reshape(T, dk)
    db, dS0 = db.ravel(), dS0.reshape(dk, dv)
    I = np.eye(dk)
    M = lambda t, s: I - sum((np.outer(k[x], k[x]) for x in range(t, s + 1)), np.zeros((dk, dk)))
    S_prev = lambda t: sum((np.outer(k[j], v[j]) for j in range(t)), np.zeros((dk, dv)))
    for j in range(T):
        want = sum((k[j] @ q[t]) * dO[t] for t in range(j, T)) + dS_T.T @ k[j]
        assert _rel(dv_[j], want) < 1e-12
        assert _rel(dq[j], sum(k[x] * (v[x] @ dO[j]) for x in range(j + 1))) < 1e-12
        want_b = sum((q[s] @ k[j]) * (v[j] @ dO[s]) for s in range(j, T)) + k[j] @ dS_T @ v[j]
        assert abs(db[j] - want_b) < 1e-12 * (1 + abs(want_b))
        want_a = sum((M(j, s) @ q[s]) * (S_prev(j) @ dO[s]) for s in range(j, T))
        want_a = want_a + ((M(j, T - 1) @ dS_T) * S_prev(j)).sum(axis=1)
        assert np.allclose(da[j], want_a, rtol=1e-12, atol=1e-12)
    want = sum(M(0, t) @ np.outer(q[t], dO[t]) for t in range(T)) + M(0, T - 1) @ dS_T
    assert _rel(dS0, want) < 1e-12


# ---------------------------------------------------------------- DeltaProduct form [DP2]


def _product(orc, q, k, v, alpha, beta, S0, signed_gate=2):
    """oracle.ckda_fwd_product on one sequence and head: q, alpha [T,dk]; k [T,nh,dk];
    v [T,nh,dv]; beta [T,nh]."""
    T, dk = q.shape
    nh, dv = k.shape[1], v.shape[2]
    o, S = orc.ckda_fwd_product(q.reshape(1, T, 1, dk), k.reshape(1, T, nh, 1, dk),
                                v.reshape(1, T, nh, 1, dv), alpha.reshape(1, T, 1, dk),
                                np.asarray(beta, float).reshape(1, T, nh, 1),
                                None if S0 is None else S0.reshape(1, 1, dk, dv),
                                signed_gate=signed_gate)
    return o.reshape(T, dv), S.reshape(dk, dv)


def pin_product_one_update(orc):
    """[DP2] One update per token is the gated delta rule itself, in every gate form."""
    rng = np.random.default_rng(40)
    T, dk, dv = 23, 5, 4
    q, k, v = rng.standard_normal((T, dk)), _unit(rng, T, dk), rng.standard_normal((T, dv))
    S0 = rng.standard_normal((dk, dv))
    for sg in range(5):
        a = rng.standard_normal((T, dk)) if sg != 2 else rng.uniform(-1, 1, (T, dk))
        b = rng.standard_normal(T) if sg != 2 else rng.uniform(0, 2, T)
        o1, S1 = _one(orc, q, k, v, a, b, S0, signed_gate=sg)
        o2, S2 = _product(orc, q, k[:, None], v[:, None], a, b[:, None], S0, signed_gate=sg)
        assert np.allclose(o1, o2, atol=1e-13) and np.allclose(S1, S2, atol=1e-13)


def pin_product_zero_second_strength(orc):
    """[DP2] With the second strength 0 the second update is the identity: the result is the
    one-update recurrence on the first key, value and strength."""
    rng = np.random.default_rng(41)
    T, dk, dv = 19, 6, 3
    q, k, v = rng.standard_normal((T, dk)), _unit(rng, T, 2, dk), rng.standard_normal((T, 2, dv))
    alpha, beta = rng.uniform(-1, 1, (T, dk)), rng.uniform(0, 2, (T, 2))
    beta[:, 1] = 0.0
    S0 = rng.standard_normal((dk, dv))
    o1, S1 = _one(orc, q, k[:, 0], v[:, 0], alpha, beta[:, 0], S0)
    o2, S2 = _product(orc, q, k, v, alpha, beta, S0)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(S1, S2, atol=1e-13)


def pin_product_idempotent_projection(orc):
    """[DP2][HH] beta = 1 with a unit key is a projection: repeating the same key and value
    changes nothing (P (P S + k v^T) + k v^T = P S + k v^T, since P k = 0)."""
    rng = np.random.default_rng(42)
    T, dk, dv = 15, 5, 4
    q, k1, v1 = rng.standard_normal((T, dk)), _unit(rng, T, dk), rng.standard_normal((T, dv))
    alpha = rng.uniform(-1, 1, (T, dk))
    S0 = rng.standard_normal((dk, dv))
    o1, S1 = _one(orc, q, k1, v1, alpha, np.ones(T), S0)
    o2, S2 = _product(orc, q, np.stack([k1, k1], 1), np.stack([v1, v1], 1), alpha,
                      np.ones((T, 2)), S0)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(S1, S2, atol=1e-12)


def pin_product_rotation(orc):
    """[DP2][HH] Two reflections (beta = 2) with unit keys at angles t1, t2 and no decay make
    the rotation R(2 (t2 - t1)); over tokens the angles add."""
    rng = np.random.default_rng(43)
    T = 9
    t1, t2 = rng.uniform(0, 2 * np.pi, T), rng.uniform(0, 2 * np.pi, T)
    k = np.stack([np.stack([np.cos(t1), np.sin(t1)], 1), np.stack([np.cos(t2), np.sin(t2)], 1)], 1)
    _, S = _product(orc, rng.standard_normal((T, 2)), k, np.zeros((T, 2, 2)), np.ones((T, 2)),
                    np.full((T, 2), 2.0), np.eye(2))
    assert np.allclose(S, _rot(2 * (t2 - t1).sum()), atol=1e-12)
    _, S1 = _product(orc, np.zeros((1, 2)), k[:1], np.zeros((1, 2, 2)), np.ones((1, 2)),
                     np.full((1, 2), 2.0), np.eye(2))
    assert np.allclose(S1, _rot(2 * (t2[0] - t1[0])), atol=1e-14)


def pin_product_explicit_matrices(orc):
    """[DP2] The product form against explicit dk x dk transitions (oracle.transition, pinned
    by its own closed forms): S <- T2 (T1 S + b1 k1 v1^T) + b2 k2 v2^T with
    T1 = (I - b1 k1 k1^T) Diag(alpha), T2 = I - b2 k2 k2^T; o = S^T q."""
    rng = np.random.default_rng(44)
    T, dk, dv = 12, 5, 3
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, 2, dk)), rng.standard_normal((T, 2, dv))
    alpha, beta = rng.uniform(-1, 1, (T, dk)), rng.uniform(0, 2, (T, 2))
    S = rng.standard_normal((dk, dv))
    o, S_T = _product(orc, q, k, v, alpha, beta, S)
    for t in range(T):
        T1 = orc.transition(k[t, 0], alpha[t], beta[t, 0])
        T2 = orc.transition(k[t, 1], np.ones(dk), beta[t, 1])
        S = T2 @ (T1 @ S + beta[t, 0] * np.outer(k[t, 0], v[t, 0])) + beta[t, 1] * np.outer(k[t, 1], v[t, 1])
        assert np.allclose(o[t], S.T @ q[t], atol=1e-12)
    assert np.allclose(S_T, S, atol=1e-12)


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
