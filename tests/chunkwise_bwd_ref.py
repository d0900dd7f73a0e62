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
"""
from __future__ import annotations

import numpy as np


def chunk_bwd_one(q, k, v, alpha, beta, S0, dO, dST, chunk: int):
    """One sequence and head.  q, k, alpha [T,dk]; v, dO [T,dv]; beta [T]; S0, dST [dk,dv].
    Returns (dq, dk, dv, dalpha, dbeta, dS0).  Every alpha must be non-zero."""
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
        A = np.tril(be[:, None] * (Kr @ Kc.T), -1)
        Tm = np.linalg.inv(np.eye(n) + A) @ np.diag(be)
        U = Tm @ (V - Kr @ S)
        S = G[-1][:, None] * (S + Kc.T @ U)
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
        M = Kr @ Kc.T
        A = np.tril(be[:, None] * M, -1)
        L = np.linalg.inv(np.eye(n) + A)
        Tm = L @ np.diag(be)
        Vp = V - Kr @ S
        U = Tm @ Vp
        P = np.tril(Qr @ Kc.T)
        Z = S + Kc.T @ U
        # reverse
        dZ = g[:, None] * dS_out
        dg = (dS_out * Z).sum(axis=1)
        dS = dZ.copy()
        dKc = U @ dZ.T
        dU = Kc @ dZ
        dQr = dOc @ S.T
        dS += Qr.T @ dOc
        dP = np.tril(dOc @ U.T)
        dU += P.T @ dOc
        dT = dU @ Vp.T
        dVp = Tm.T @ dU
        gv[t0:t1] += dVp
        dKr = -dVp @ S.T
        dS -= Kr.T @ dVp
        dL = dT * be[None, :]
        dbe = (L * dT).sum(axis=0)
        dA = np.tril(-L.T @ dL @ L.T, -1)
        dbe += (dA * M).sum(axis=1)
        dM = be[:, None] * dA
        dKr += dM @ Kc
        dKc += dM.T @ Kr
        dQr += dP @ Kc
        dKc += dP.T @ Qr
        gk[t0:t1] += dKr * G + dKc / G
        gq[t0:t1] += dQr * G
        dG = dKr * K + dQr * Q - dKc * Kc / G
        dG[-1] += dg
        suffix = np.cumsum((dG * G)[::-1], axis=0)[::-1]
        ga[t0:t1] += suffix / al
        gb[t0:t1] += dbe
        dS_out = dS
    return gq, gk, gv, ga, gb, dS_out
