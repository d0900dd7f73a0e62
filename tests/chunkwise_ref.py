"""Independent fp64 numpy statement of the chunkwise UT (WY) form.

Test infrastructure: used only to cross-check the sequential oracle (the two
share no code).  Gates are given as raw alpha in [-1, 1] and beta, so no
activation arithmetic is involved.

Within a chunk with incoming state S0 and positions r = 0..n-1, write
g(r, j) = prod_{s=j+1..r} alpha_s  (per channel; 1 when r == j) and
G_r = prod_{s<=r} alpha_s.  The delta-rule recurrence
S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
("Complex KDA" review, section "Diagonal-plus-rank-one (DPR1) transition";
the review states it keeps WY chunk-wise parallelism) unrolls to

  A[r, j] = beta_r sum_c k_rc k_jc g(r, j)_c        (j < r)
  P[r, j] =        sum_c q_rc k_jc g(r, j)_c        (j <= r)
  Tm      = (I + A)^{-1} Diag(beta)
  U       = Tm V - Tm (K * G) S0
  O       = (Q * G) S0 + P U
  S_n     = Diag(G_{n-1}) S0 + (K * g(n-1, .))^T U

The ratios g are formed as explicit products, so zero gates need no care.
"""
from __future__ import annotations

import numpy as np


def _ratio_table(alpha: np.ndarray) -> np.ndarray:
    """g[r, j, c] = prod_{s=j+1..r} alpha[s, c] for j <= r, 0 above the diagonal."""
    n, d = alpha.shape
    g = np.zeros((n, n, d))
    for j in range(n):
        acc = np.ones(d)
        g[j, j] = acc
        for r in range(j + 1, n):
            acc = acc * alpha[r]
            g[r, j] = acc
    return g


def chunk_fwd_one(q, k, v, alpha, beta, S0, chunk: int):
    """One sequence, one head.  q, k, alpha [T,dk]; v [T,dv]; beta [T]; S0 [dk,dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T, dv))
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        n = t1 - t0
        Q, K, V = q[t0:t1], k[t0:t1], v[t0:t1]
        al, be = alpha[t0:t1], beta[t0:t1]
        g = _ratio_table(al)                       # [n, n, dk]
        G = np.cumprod(al, axis=0)                  # G[r] = prod_{s<=r} alpha_s
        A = np.einsum("rc,jc,rjc->rj", K, K, g) * be[:, None]
        A = np.tril(A, -1)
        P = np.tril(np.einsum("rc,jc,rjc->rj", Q, K, g))
        Tm = np.linalg.inv(np.eye(n) + A) @ np.diag(be)
        W = Tm @ (K * G)
        U = Tm @ V - W @ S
        o[t0:t1] = (Q * G) @ S + P @ U
        tail = g[n - 1]                             # g(n-1, j) for every j
        S = np.diag(G[n - 1]) @ S + (K * tail).T @ U
    return o, S
