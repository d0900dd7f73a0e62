"""The chunkwise (UT-form) backward, stated independently in numpy
(``chunkwise_bwd_ref.py``), equals the sequential oracle's backward in fp64: the algebra a
chunkwise backward kernel computes, checked before any such kernel exists.  CPU only."""
import numpy as np
import pytest

import oracle
from chunkwise_bwd_ref import chunk_bwd_one


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


@pytest.mark.parametrize("chunk", [1, 2, 16, 64])
@pytest.mark.parametrize("T,zero_ends", [(150, False), (64, True), (7, False)])
def test_chunkwise_backward_equals_sequential(chunk, T, zero_ends):
    args = _case(T, 8, 6, seed=T + chunk, zero_ends=zero_ends)
    ref = _oracle(*args)
    got = chunk_bwd_one(*args, chunk)
    for name, g, r in zip(("dq", "dk", "dv", "dalpha", "dbeta", "dS0"), got, ref):
        n = np.linalg.norm(r)
        err = np.linalg.norm(g.reshape(-1) - r) / (n if n > 0 else 1.0)
        assert err < 1e-11, (name, err)
