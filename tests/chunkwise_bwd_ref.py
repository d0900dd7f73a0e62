"""Independent fp64 numpy statement of the chunkwise (UT-form) BACKWARD.

Test infrastructure: used only to check the algebra a chunkwise backward kernel would
compute, against the sequential oracle's backward (the two share no code).  Gates are given
raw (alpha in [-1, 1], beta), so the result is the gradient with respect to alpha and beta
themselves.

Forward of one chunk with incoming state S (rows r = 0..C-1, per-channel products
G_r = prod_{s<=r} alpha_s, written G):
  Kr = K*G   Qr = Q*G   Kc = K/G
  A  = tril(Diag(beta) Kr Kc^T, -1)      P = tril(Qr Kc^T)
  L  = (I + A)^{-1}    T = L Diag(beta)
  V' = V - Kr S        U = T V'
  O  = Qr S + P U      S' = Diag(g) Z,  Z = S + Kc^T U,  g = G_{C-1}
("Complex KDA" review, section "Diagonal-plus-rank-one (DPR1) transition": the DPR1
transition keeps the WY chunk-wise form; the reverse below is its plain chain rule.)

Backward, given dO and dS' (the gradient of the chunk's outgoing state), in reverse order:
  S' = Diag(g) Z:      dZ = Diag(g) dS',         dg_i = sum_j dS'_ij Z_ij
  Z = S + Kc^T U:      dS = dZ,  dKc = U dZ^T,   dU = Kc dZ
  O = Qr S + P U:      dQr = dO S^T,  dS += Qr^T dO,  dP = tril(dO U^T),  dU += P^T dO
  U = T V':            dT = dU V'^T,  dV' = T^T dU
  V' = V - Kr S:       dV = dV',  dKr = -dV' S^T,  dS -= Kr^T dV'
  T = L Diag(beta):    dL = dT Diag(beta),  dbeta_j = sum_r L_rj dT_rj
  L = (I + A)^{-1}:    dA = -L^T dL L^T, kept strictly lower
  A = tril(Diag(beta) M, -1), M = Kr Kc^T:
                       dbeta_r += sum_{j<r} dA_rj M_rj,  dM = Diag(beta) dA (strictly lower)
                       dKr += dM Kc,  dKc += dM^T Kr
  P = tril(Qr Kc^T):   dQr += dP Kc,  dKc += dP^T Qr
  Kr, Qr, Kc:          dK = dKr*G + dKc/G,  dQ = dQr*G,
                       dG = dKr*K + dQr*Q - dKc*Kc/G,  dG_{C-1} += dg
  G_r = prod_{s<=r} alpha_s:  dalpha_s = (sum_{r>=s} dG_r G_r) / alpha_s   (alpha_s != 0)
The chunks are walked last to first with dS' of a chunk = dS of the next one.

The last line, the "factorised" gate gradient, adds terms that cancel pairwise: with K/G large
where the chunk's products decay, rounding of those terms leaves an error far above their
sum.  ``dlog_alpha_pairwise`` keeps only the terms that survive the cancellation (pairs of
rows straddling s, each weighted by a gate ratio of size <= 1), the same value exactly.
"""
from __future__ import annotations

import numpy as np


def _ratio_table(alpha):
    """g[t, j, c] = prod_{s=j+1..t} alpha[s, c] for j <= t (explicit products), 0 above."""
    n, d = alpha.shape
    g = np.zeros((n, n, d))
    for j in range(n):
        acc = np.ones(d)
        g[j, j] = acc
        for t in range(j + 1, n):
            acc = acc * alpha[t]
            g[t, j] = acc
    return g


def dlog_alpha_pairwise(Q, K, S, dO, dVp, dM, dP, dS_out, U, G, g_tab, mm=np.matmul):
    """Gradient with respect to log|alpha_s| of one chunk, formed only from terms of moderate
    size.  In the suffix sum of (dKr Kr + dQr Qr - dKc Kc) every pair (t, j) with both rows
    on the same side of s cancels; what remains is
      sum_{t>=s} [(-dV'_t S^T) * Kr_t + (dO_t S^T) * Qr_t]               state read, G <= 1
      + sum_{t>=s>j} (dM_tj K_t K_j + dP_tj Q_t K_j) g(t,j)             intra-chunk pairs
      + sum_{t<s} (K_t g(C-1,t)) * (dS' U_t^T)                          state write
      + g * rowsum(dS' * S)                                             carried state
    with every gate factor a product of |alpha| <= 1 over the rows it spans."""
    n, d = K.shape
    Kr, Qr = K * G, Q * G
    read = -mm(dVp, S.T) * Kr + mm(dO, S.T) * Qr                       # [n, d]
    # pairs: W[t, j, c] for j < t
    W = (dM[:, :, None] * K[:, None, :] * K[None, :, :]
         + dP[:, :, None] * Q[:, None, :] * K[None, :, :]) * g_tab
    W = W * np.tril(np.ones((n, n)), -1)[:, :, None]
    write = K * g_tab[n - 1] * mm(U, dS_out.T)                         # [n, d] rows t
    carry = G[n - 1] * (dS_out * S).sum(axis=1)                        # [d]
    out = np.zeros((n, d))
    for s_ in range(n):
        out[s_] = (read[s_:].sum(axis=0) + W[s_:, :s_].sum(axis=(0, 1))
                   + write[:s_].sum(axis=0) + carry)
    return out


def chunk_bwd_one(q, k, v, alpha, beta, S0, dO, dST, chunk: int, gate_grad: str = "factorised",
                  mm=np.matmul):
    """One sequence and head.  q, k, alpha [T,dk]; v, dO [T,dv]; beta [T]; S0, dST [dk,dv].
    Returns (dq, dk, dv, dalpha, dbeta, dS0).  Every alpha must be non-zero.  ``gate_grad``:
    "factorised" forms dalpha from the suffix sums of dG G; "pairwise" from
    ``dlog_alpha_pairwise`` (the same value in exact arithmetic, without the cancellation).
    ``mm`` computes every matrix product (a test passes one with rounded operands)."""
    T, dk = q.shape
    dv = v.shape[1]
    # forward, keeping each chunk's incoming state
    S = np.array(S0, dtype=np.float64, copy=True)
    starts = list(range(0, T, chunk))
    S_in = []
    for t0 in starts:
        t1 = min(T, t0 + chunk)
        S_in.append(S.copy())
        K, V = k[t0:t1], v[t0:t1]
        al, be = alpha[t0:t1], beta[t0:t1]
        G = np.cumprod(al, axis=0)
        n = t1 - t0
        Kr, Kc = K * G, K / G
        A = np.tril(be[:, None] * mm(Kr, Kc.T), -1)
        Tm = mm(np.linalg.inv(np.eye(n) + A), np.diag(be))
        U = mm(Tm, V - mm(Kr, S))
        S = G[-1][:, None] * (S + mm(Kc.T, U))
    gq, gk, gv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ga, gb = np.zeros_like(alpha), np.zeros_like(beta)
    dS_out = np.array(dST, dtype=np.float64, copy=True)
    for ci in range(len(starts) - 1, -1, -1):
        t0 = starts[ci]
        t1 = min(T, t0 + chunk)
        n = t1 - t0
        S = S_in[ci]
        Q, K, V = q[t0:t1], k[t0:t1], v[t0:t1]
        al, be, dOc = alpha[t0:t1], beta[t0:t1], dO[t0:t1]
        # recompute the chunk's forward quantities
        G = np.cumprod(al, axis=0)
        g = G[-1]
        Kr, Qr, Kc = K * G, Q * G, K / G
        M = mm(Kr, Kc.T)
        A = np.tril(be[:, None] * M, -1)
        L = np.linalg.inv(np.eye(n) + A)
        Tm = mm(L, np.diag(be))
        Vp = V - mm(Kr, S)
        U = mm(Tm, Vp)
        P = np.tril(mm(Qr, Kc.T))
        Z = S + mm(Kc.T, U)
        # reverse
        dZ = g[:, None] * dS_out
        dg = (dS_out * Z).sum(axis=1)
        dS = dZ.copy()
        dKc = mm(U, dZ.T)
        dU = mm(Kc, dZ)
        dQr = mm(dOc, S.T)
        dS += mm(Qr.T, dOc)
        dP = np.tril(mm(dOc, U.T))
        dU += mm(P.T, dOc)
        dT = mm(dU, Vp.T)
        dVp = mm(Tm.T, dU)
        gv[t0:t1] += dVp
        dKr = -mm(dVp, S.T)
        dS -= mm(Kr.T, dVp)
        dL = dT * be[None, :]
        dbe = (L * dT).sum(axis=0)
        dA = np.tril(-mm(mm(L.T, dL), L.T), -1)
        dbe += (dA * M).sum(axis=1)
        dM = be[:, None] * dA
        dKr += mm(dM, Kc)
        dKc += mm(dM.T, Kr)
        dQr += mm(dP, Kc)
        dKc += mm(dP.T, Qr)
        gk[t0:t1] += dKr * G + dKc / G
        gq[t0:t1] += dQr * G
        dG = dKr * K + dQr * Q - dKc * Kc / G
        dG[-1] += dg
        if gate_grad == "pairwise":
            ga[t0:t1] += dlog_alpha_pairwise(Q, K, S, dOc, dVp, dM, dP, dS_out, U, G,
                                             _ratio_table(al), mm) / al
        else:
            suffix = np.cumsum((dG * G)[::-1], axis=0)[::-1]
            ga[t0:t1] += suffix / al
        gb[t0:t1] += dbe
        dS_out = dS
    return gq, gk, gv, ga, gb, dS_out
