"""The chunkwise (UT-form) backward, stated independently in numpy
(``chunkwise_bwd_ref.py``), equals the sequential oracle's backward in fp64: the algebra a
chunkwise backward kernel computes, checked before any such kernel exists.  With tf32
operands in every matrix product it stays within the bf16 tolerance provided the gate
gradient is formed pairwise (see the reference's docstring).  CPU only."""
import numpy as np
import pytest

import oracle
from chunkwise_bwd_ref import chunk_bwd_one
from helpers import TOL_BF16, f64
from linear_rnn_ckda_b200 import synth
from test_chunk_algebra import tf32_nearest


def _case(T, dk, dv, seed, zero_ends=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    alpha = rng.uniform(0.3, 1.0, (T, dk)) * rng.choice([-1.0, 1.0], (T, dk))   # signed, non-zero
    beta = rng.uniform(0.0, 2.0, T)
    S0 = np.zeros((dk, dv)) if zero_ends else rng.standard_normal((dk, dv))
    dO = rng.standard_normal((T, dv))
    dST = np.zeros((dk, dv)) if zero_ends else rng.standard_normal((dk, dv))
    return q, k, v, alpha, beta, S0, dO, dST


def _oracle(q, k, v, alpha, beta, S0, dO, dST):
    T, dk = q.shape
    dv = v.shape[1]
    r = lambda x, *s: x.reshape(*s)
    out = oracle.ckda_bwd(r(q, 1, T, 1, dk), r(k, 1, T, 1, dk), r(v, 1, T, 1, dv),
                          r(alpha, 1, T, 1, dk), r(beta, 1, T, 1), r(S0, 1, 1, dk, dv),
                          dO=r(dO, 1, T, 1, dv), dS_T=r(dST, 1, 1, dk, dv), signed_gate=2, threads=1)
    return [x.reshape(-1) for x in out]


@pytest.mark.parametrize("gate_grad", ["factorised", "pairwise"])
@pytest.mark.parametrize("chunk", [1, 2, 16, 64])
@pytest.mark.parametrize("T,zero_ends", [(150, False), (64, True), (7, False)])
def test_chunkwise_backward_equals_sequential(chunk, T, zero_ends, gate_grad):
    args = _case(T, 8, 6, seed=T + chunk, zero_ends=zero_ends)
    ref = _oracle(*args)
    got = chunk_bwd_one(*args, chunk, gate_grad)
    for name, g, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), got, ref):
        n = np.linalg.norm(r)
        err = np.linalg.norm(g.reshape(-1) - r) / (n if n > 0 else 1.0)
        assert err < 1e-11, (name, err)


# ---------------------------------------------------------------- tf32 operand plan
def _mm_tf32(a, b):
    """A matrix product with tf32 operands (round to nearest) and an fp32 result."""
    a32 = tf32_nearest(np.asarray(a, np.float32)).astype(np.float64)
    b32 = tf32_nearest(np.asarray(b, np.float32)).astype(np.float64)
    return (a32 @ b32).astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("base,form", [(synth.KDA_STD, 0), (synth.CKDA_SPREAD, 1)],
                         ids=["kda_std", "ckda_spread"])
def test_tf32_operand_plan(base, form):
    """bf16 inputs at the full head size (d = 128, chunk 64, a ragged tail) with every matrix
    product on tf32 operands: with the pairwise gate gradient every gradient stays at half the
    bf16 tolerance or below.  The factorised gate gradient sums terms that cancel when the
    chunk's gate products decay (K/G grows as G shrinks), so on the spread workload its
    error is several times the pairwise one."""
    w = base.with_(B=1, T=2 * 64 + 45, H=1, signed_gate=form, o_dtype="f32")
    inp = synth.make_prefill(w, seed=7)
    q, k, v, a, b = (f64(inp[x])[0, :, 0] for x in "qkvab")
    alpha, beta = oracle.gates(a, b, form)
    T, d = q.shape
    rng = np.random.default_rng(1)
    S0 = f64(inp["S0"])[0, 0] if inp["S0"] is not None else np.zeros((d, d))
    dO = rng.standard_normal((T, d))
    dST = rng.standard_normal((d, d)) * 0.02
    ref = _oracle(q, k, v, alpha, beta, S0, dO, dST)
    errs = {}
    for gate_grad in ("pairwise", "factorised"):
        got = chunk_bwd_one(q, k, v, alpha, beta, S0, dO, dST, 64, gate_grad, mm=_mm_tf32)
        errs[gate_grad] = [np.linalg.norm(g.reshape(-1) - r) / np.linalg.norm(r)
                           for g, r in zip(got, ref)]
    assert max(errs["pairwise"]) < TOL_BF16 / 2, errs["pairwise"]
    if form == 1:
        assert errs["factorised"][3] > 5 * errs["pairwise"][3], (errs["factorised"][3],
                                                                 errs["pairwise"][3])


def test_state_gradient_recurrence():
    """The backward's only sequential dependency, written with the forward's chunk tiles:
    dS_prev = dZ - Kr^T T^T (Kc dZ) + (Qr^T dO - Kr^T T^T P^T dO), dZ = Diag(g) dS'; equal
    to the state gradient of the step-by-step reverse (chunkwise_bwd_ref's order)."""
    rng = np.random.default_rng(2)
    n, dk, dv = 16, 6, 5
    Q, K = rng.standard_normal((n, dk)), rng.standard_normal((n, dk))
    alpha = rng.uniform(0.4, 1, (n, dk)) * rng.choice([-1.0, 1.0], (n, dk))
    beta = rng.uniform(0, 2, n)
    dO, dS_out = rng.standard_normal((n, dv)), rng.standard_normal((dk, dv))
    G = np.cumprod(alpha, axis=0)
    Kr, Qr, Kc = K * G, Q * G, K / G
    A = np.tril(beta[:, None] * (Kr @ Kc.T), -1)
    Tm = np.linalg.inv(np.eye(n) + A) @ np.diag(beta)
    P = np.tril(Qr @ Kc.T)
    dZ = G[-1][:, None] * dS_out
    # step-by-step reverse: dU from the state write and the output, dV' = T^T dU
    dVp = Tm.T @ (Kc @ dZ + P.T @ dO)
    step = dZ + Qr.T @ dO - Kr.T @ dVp
    recurrence = dZ - Kr.T @ (Tm.T @ (Kc @ dZ)) + (Qr.T @ dO - Kr.T @ (Tm.T @ (P.T @ dO)))
    assert np.allclose(recurrence, step, rtol=1e-12, atol=1e-12 * np.abs(step).max())
