"""The algebra the tensor-core prefill's segment plan rests on, checked on the fp64 oracle.

Over a stretch of tokens the recurrence S_t = (I - b_t k_t k_t^T) Diag(alpha_t) S_{t-1} +
b_t k_t v_t^T (CKDA review, section "Diagonal-plus-rank-one (DPR1) transition") is affine in
the state it starts from: S_end = A S_in + B, with A the ordered product of the stretch's
transitions and B the end state from S_in = 0.  A is the end state of the same walk from
S_in = I with every v_t = 0.  The plan runs a cut sequence's segments from 0 and from I,
chains X_s <- Y_s X_{s-1} + X_s and reruns each segment from its chained state; here that
chain, written on the oracle, reproduces the uncut sequence's outputs and end state, and the
affine identity holds for any starting state."""
import numpy as np
import pytest

import oracle

D = 8   # dk = dv: A is a state-shaped [dk][dk] matrix, as in the kernels (dk = dv = 128)


def _inputs(T, H, sg, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, H, D))
    k = rng.standard_normal((1, T, H, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, D))
    # slow gates (|alpha| ~ 0.98), so that a stretch's transition product does not vanish
    # and the orientation of A S_in shows; CKDA gates with random signs
    a = rng.standard_normal((1, T, H, D)) * 0.5 + 4.0
    if sg:
        a *= np.where(rng.random(a.shape) < 0.5, 1.0, -1.0)
    b = rng.standard_normal((1, T, H))
    return q, k, v, a, b


def _run(x, lo, hi, S0, sg, zero_v=False):
    q, k, v, a, b = (y[:, lo:hi] for y in x)
    if zero_v:
        v = np.zeros_like(v)
    return oracle.ckda_fwd(q, k, v, a, b, S0, signed_gate=sg)


@pytest.mark.parametrize("sg", [0, 1], ids=["kda", "ckda"])
def test_segment_map_is_affine(sg):
    """End state from any S_in = (walk from I, v = 0) S_in + (walk from 0)."""
    H, T = 2, 37
    x = _inputs(T, H, sg, seed=200 + sg)
    eye = np.broadcast_to(np.eye(D), (1, H, D, D)).copy()
    _, A = _run(x, 0, T, eye, sg, zero_v=True)
    _, B = _run(x, 0, T, np.zeros((1, H, D, D)), sg)
    rng = np.random.default_rng(210 + sg)
    for _ in range(3):
        S_in = rng.standard_normal((1, H, D, D))
        _, S = _run(x, 0, T, S_in, sg)
        assert np.allclose(S, A @ S_in + B, rtol=1e-11, atol=1e-12)
    # A is not negligible, far from the identity and not symmetric, and B is not zero: the
    # check has something to check (S_in A + B or A^T S_in + B would fail it)
    assert np.abs(A).max() > 1e-2 and np.abs(A - eye).max() > 1e-2 and np.abs(B).max() > 1e-2
    assert np.abs(A - np.swapaxes(A, -1, -2)).max() > 1e-2


@pytest.mark.parametrize("sg", [0, 1], ids=["kda", "ckda"])
@pytest.mark.parametrize("cuts", [(30, 60), (13, 50, 77)])
def test_segment_chain_reproduces_the_sequence(sg, cuts):
    """X_0 from S0; X_s from 0 and Y_s from I (v = 0) for the middle segments; the chain
    X_s <- Y_s X_{s-1} + X_s; every segment rerun from its chained state gives the uncut
    walk's outputs row for row and its end state."""
    H, T = 2, 90
    x = _inputs(T, H, sg, seed=220 + sg + len(cuts))
    S0 = np.random.default_rng(230).standard_normal((1, H, D, D)) * 0.1
    o_ref, S_ref = _run(x, 0, T, S0, sg)
    bounds = (0,) + tuple(cuts) + (T,)
    m = len(bounds) - 1
    eye = np.broadcast_to(np.eye(D), (1, H, D, D)).copy()
    X = [_run(x, bounds[0], bounds[1], S0, sg)[1]]
    for s in range(1, m - 1):
        _, Xs = _run(x, bounds[s], bounds[s + 1], np.zeros((1, H, D, D)), sg)
        _, Ys = _run(x, bounds[s], bounds[s + 1], eye, sg, zero_v=True)
        X.append(Ys @ X[s - 1] + Xs)
    o_parts = [_run(x, bounds[0], bounds[1], S0, sg)[0]]
    S_end = None
    for s in range(1, m):
        o_s, S_end = _run(x, bounds[s], bounds[s + 1], X[s - 1], sg)
        o_parts.append(o_s)
    o = np.concatenate(o_parts, axis=1)
    assert np.allclose(o, o_ref, rtol=1e-10, atol=1e-11)
    assert np.allclose(S_end, S_ref, rtol=1e-10, atol=1e-11)
