"""CPU statement of the tensor-core chunk kernel's algebra and operand precision,
checked against the sequential fp64 oracle.

Test infrastructure (numpy only; shares no code with the CUDA path).  The
tensor-core prefill does not follow the textbook WY form step by step: it
regroups U = T (V - (K*G) S), inverts (I + A) in 16-row blocks with the
off-diagonal blocks applied as three corrections, keeps K*G^{-1} with the
final G folded in afterwards, and rounds every tensor-core operand to tf32.
Each of those choices is an algebraic identity or a precision decision; this
file states them in numpy and checks

  * the identities exactly (fp64, no rounding) against the delta-rule
    recurrence ("Complex KDA" review, section "Diagonal-plus-rank-one (DPR1)
    transition"), on several chunks with a ragged tail;
  * the operand plan (tf32 operands rounded to nearest or truncated where the
    kernel reads them from tensor memory, fp32 accumulation, fp32 gate
    products) against the 2e-3 bf16 tolerance, with margin;
  * the integer tf32 rounding ((bits + 0x1000) & ~0x1FFF) against the
    definition of round-to-nearest, ties away from zero, onto the tf32 grid.

Both ways of applying (I + A)^{-1} are checked: the fused kernel's
block-diagonal product plus three corrections, and the full T assembled
from the same blocks and applied in one product (the form a state pass that
reads T computed elsewhere would use).

The tensor core's own accumulation order is not specified; the emulation
forms each product exactly and rounds it to fp32 once, which is the most
favourable accumulation, so the checks on the plan keep a factor of two of
margin below the tolerance the GPU tests use.
"""
from __future__ import annotations

import numpy as np
import pytest

from helpers import TOL_BF16, f64, oracle_prefill, rel, unit_rows
from linear_rnn_ckda_b200 import synth

import oracle

C = 64          # chunk
NB = 16         # rows of one block of the solve


# ------------------------------------------------------------------ tf32 grid
def tf32_nearest(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the tf32 grid (10 explicit mantissa bits, fp32's exponent
    range), to nearest with ties away from zero; values past the largest tf32 by half a
    step or more become infinities.  Written from the definition: the two grid neighbours
    of |x| and a comparison of distances in float64."""
    x = np.asarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    sign = bits & np.uint32(0x80000000)
    mag = bits & np.uint32(0x7FFFFFFF)
    low = mag & np.uint32(0xFFFFE000)                       # neighbour toward zero
    high = low + np.uint32(0x2000)                          # neighbour away from zero
    lv = low.view(np.float32).astype(np.float64)
    hv = high.view(np.float32).astype(np.float64)
    hv = np.where(np.isinf(hv), 2.0 ** 128, hv)             # unbounded-exponent value of inf
    xv = mag.view(np.float32).astype(np.float64)
    up = (hv - xv) <= (xv - lv)                             # ties go away from zero
    out = np.where(up, high, low) | sign
    finite = mag < np.uint32(0x7F800000)
    return np.where(finite, out, bits).view(np.float32)


def tf32_trunc(x: np.ndarray) -> np.ndarray:
    """The tf32 value a tensor-core read of an fp32 word takes (low 13 bits dropped)."""
    x = np.asarray(x, dtype=np.float32)
    return (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def tf32_integer_rounding(x: np.ndarray) -> np.ndarray:
    """The kernel's integer form of round-to-nearest tf32."""
    x = np.asarray(x, dtype=np.float32)
    with np.errstate(over="ignore"):
        b = (x.view(np.uint32) + np.uint32(0x1000)) & np.uint32(0xFFFFE000)
    return b.view(np.float32)


def test_integer_tf32_rounding_matches_definition():
    rng = np.random.default_rng(11)
    # random bit patterns over every finite float, plus ties, carries into the exponent,
    # subnormals, zeros and the overflow boundary
    bits = rng.integers(0, 0x7F800000, size=200_000, dtype=np.uint64).astype(np.uint32)
    special = np.array([0x00000000, 0x00000001, 0x00000FFF, 0x00001000, 0x00001FFF,
                        0x00002000, 0x00003000, 0x007FF000, 0x007FFFFF, 0x3F800FFF,
                        0x3F801000, 0x3F802FFF, 0x3F803000, 0x3FFFF000, 0x3FFFEFFF,
                        0x7F7FE000, 0x7F7FEFFF, 0x7F7FF000, 0x7F7FFFFF], dtype=np.uint32)
    bits = np.concatenate([bits, special])
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
    x = bits.view(np.float32)
    want = tf32_nearest(x)
    got = tf32_integer_rounding(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # the grid itself: 10 explicit mantissa bits, so 1 + 2^-10 is on it and 1 + 2^-11 ties up
    one = np.float32(1.0)
    assert tf32_nearest(np.float32(1 + 2.0 ** -10)) == np.float32(1 + 2.0 ** -10)
    assert tf32_nearest(np.float32(1 + 2.0 ** -11)) == np.float32(1 + 2.0 ** -10)
    assert tf32_nearest(np.float32(1 + 2.0 ** -12)) == one
    assert np.isinf(tf32_nearest(np.float32(np.finfo(np.float32).max)))


# ------------------------------------------------------------------ one (sequence, head)
def _gates_f32(a: np.ndarray, form: int):
    """Gate and inverse gate per element in fp32 by the kernel's formulas:
    KDA sigma(a) = 1 / (1 + e^{-a}) with inverse 1 + e^{-a}; CKDA 2 sigma(a) - 1 =
    sign(a) (1 - e^{-|a|}) / (1 + e^{-|a|}) with the ratio upside down as its inverse."""
    a = a.astype(np.float32)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        if form == 0:
            e = np.exp(-a)
            ial = np.float32(1) + e
            al = np.float32(1) / ial
        else:
            e = np.exp(-np.abs(a))
            num, den = np.float32(1) - e, np.float32(1) + e
            r = np.copysign(np.float32(1) / (num * den), a)
            al, ial = num * (num * r), den * (den * r)
    return al.astype(np.float32), ial.astype(np.float32)


def _running_products(al: np.ndarray) -> np.ndarray:
    """Per channel, products G_t of the gates of rows 0..t in the kernel's order: a running
    product inside each 8-row group, times the product of the earlier groups' totals."""
    G = np.empty_like(al)
    mult = np.ones(al.shape[1], dtype=al.dtype)
    with np.errstate(over="ignore"):      # inverse gates of a decayed chunk overflow fp32
        for g0 in range(0, al.shape[0], 8):
            run = np.ones(al.shape[1], dtype=al.dtype)
            for r in range(g0, min(g0 + 8, al.shape[0])):
                run = run * al[r]
                G[r] = run * mult
            mult = mult * run
    return G


class _Plan:
    """Rounding of operands and products: exact (fp64) or the kernel's (tf32 operands,
    fp32 results)."""

    def __init__(self, tf32: bool):
        self.tf32 = tf32
        self.dt = np.float32 if tf32 else np.float64

    def smem(self, x):          # an operand written to shared memory
        return tf32_nearest(x.astype(np.float32)) if self.tf32 else x

    def tmem(self, x):          # an fp32 word in tensor memory read as an operand
        return tf32_trunc(x) if self.tf32 else x

    def mma(self, a, b, acc=None):
        p = a.astype(np.float64) @ b.astype(np.float64)
        if acc is not None:
            p = p + acc.astype(np.float64)
        return p.astype(self.dt)


def _block_solve(A, plan: _Plan):
    """Diagonal-block inverses X_i = D_i^{-1} (D_i = I + A_ii) and M_ij = X_i A_ij by
    forward substitution of 16 rows, in the working precision."""
    dt = plan.dt
    nb = C // NB
    X, M = {}, {}
    for i in range(nb):
        D = np.eye(NB, dtype=dt) + A[i * NB:(i + 1) * NB, i * NB:(i + 1) * NB]
        rhs = {i: np.eye(NB, dtype=dt)}
        for j in range(i):
            rhs[j] = A[i * NB:(i + 1) * NB, j * NB:(j + 1) * NB]
        for j, R in rhs.items():
            Y = np.zeros((NB, NB), dtype=dt)
            for r in range(NB):
                Y[r] = R[r] - D[r, :r] @ Y[:r]         # unit diagonal
            if j == i:
                X[i] = Y
            else:
                M[(i, j)] = Y
    return X, M


def _full_T(Xi, M, be, dt):
    """(I + A)^{-1} Diag(beta) assembled from the block solve: diagonal blocks X_i Diag(beta_i),
    T_ij = -sum_{k=j}^{i-1} M_ik T_kj below them (three dependency levels)."""
    Tf = np.zeros((C, C), dtype=dt)
    for i in range(C // NB):
        sl = slice(i * NB, (i + 1) * NB)
        Tf[sl, sl] = Xi[i] * be[sl][None, :]
    for lev in (1, 2, 3):
        for j in range(C // NB - lev):
            i = j + lev
            acc = np.zeros((NB, NB))
            for kk in range(j, i):
                acc += M[(i, kk)].astype(np.float64) @ Tf[kk * NB:(kk + 1) * NB,
                                                           j * NB:(j + 1) * NB].astype(np.float64)
            Tf[i * NB:(i + 1) * NB, j * NB:(j + 1) * NB] = (-acc).astype(dt)
    return Tf


def chunk_kernel_form(q, k, v, a, b, S0, form: int, plan: _Plan, solve: str = "corrections"):
    """One sequence and head through the kernel's steps.  q, k, a [T,d]; v [T,dv]; b [T]
    (logits); S0 [d,dv].  Returns (o [T,dv], S_T [d,dv]).  ``solve`` = "corrections": U from the
    block-diagonal part of T and three corrections (the fused kernel); "full": U from
    the full T in one product (a state pass that reads T precomputed elsewhere)."""
    dt = plan.dt
    T, dk = q.shape
    if plan.tf32:
        al_all, ial_all = _gates_f32(a, form)
        beta_all = (1 if form == 0 else 2) / (1 + np.exp(-b.astype(np.float32)))
        beta_all = beta_all.astype(np.float32)
    else:
        al_all, beta_all = oracle.gates(a, b, form)
        ial_all = 1.0 / al_all
    S = S0.astype(dt).copy()
    o = np.zeros((T, v.shape[1]), dtype=dt)
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        # rows past the end: zero inputs, unit gate, zero strength
        pad = lambda x, fill: np.concatenate([x[t0:t0 + n].astype(dt),
                                              np.full((C - n,) + x.shape[1:], fill, dt)])
        Q, K, V = pad(q, 0), pad(k, 0), pad(v, 0)
        al, ial, be = pad(al_all, 1), pad(ial_all, 1), pad(beta_all, 0)
        G, IG = _running_products(al), _running_products(ial)
        gl = np.abs(G[C - 1])
        if not np.all((gl >= 2.0 ** -100) & (gl <= 2.0 ** 100)):
            # outside the factorised path's range: this chunk runs token by token, with the
            # gates from their definition
            ex_al, ex_be = oracle.gates(a[t0:t0 + n], b[t0:t0 + n], form)
            for r in range(n):
                kt, qt = k[t0 + r].astype(dt), q[t0 + r].astype(dt)
                S = (S * ex_al[r].astype(dt)[:, None]).astype(dt)
                S = (S + dt(ex_be[r]) * np.outer(kt, v[t0 + r].astype(dt) - kt @ S)).astype(dt)
                o[t0 + r] = qt @ S
            continue
        Kr, Qr, Kc = plan.smem(K * G), plan.smem(Q * G), plan.smem(K * IG)
        # (1) [A; P] = [Kr; Qr] Kc^T;  (a) [X | O] = [Kr; Qr] S
        A = np.tril(plan.mma(Kr, Kc.T) * be[:, None], -1).astype(dt)
        P = plan.smem(np.tril(plan.mma(Qr, Kc.T)))
        St = plan.tmem(S)
        X, Oc = plan.mma(Kr, St), plan.mma(Qr, St)
        # V' = V - X as a rounded hi part and its remainder
        Vp = (V - X).astype(dt)
        hi = plan.smem(Vp)
        lo = plan.tmem((Vp - hi).astype(dt))
        # (c) U = Tb V' with Tb = blockdiag(X_i) Diag(beta); corrections U_i -= M_ij U_j
        Xi, M = _block_solve(A, plan)
        if solve == "full":
            Tt = plan.smem(_full_T(Xi, M, be, dt))
            U = plan.mma(Tt, lo, plan.mma(Tt, hi))
        else:
            Tb = np.zeros((C, C), dtype=dt)
            for i in range(C // NB):
                sl = slice(i * NB, (i + 1) * NB)
                Tb[sl, sl] = Xi[i] * be[sl][None, :]
            Tb = plan.smem(Tb)
            U = plan.mma(Tb, lo, plan.mma(Tb, hi))
            for j in range(C // NB - 1):
                Uj = plan.tmem(U[j * NB:(j + 1) * NB])
                for i in range(j + 1, C // NB):
                    U[i * NB:(i + 1) * NB] = plan.mma(-plan.smem(M[(i, j)]), Uj,
                                                      U[i * NB:(i + 1) * NB])
        # (d) O += P U;  S += Kc^T U, then the columns scaled by G_{C-1}
        Ut = plan.tmem(U)
        o[t0:t0 + n] = plan.mma(P, Ut, Oc)[:n]
        S = plan.mma(Kc.T, Ut, S)
        S = (S * G[C - 1][:, None]).astype(dt)
    return o, S


def _units(inp):
    q, k, v, a = (f64(inp[x]) for x in "qkva")
    b = f64(inp["b"])
    S0 = inp.get("S0")
    B, T, H, dk = q.shape
    for n in range(B):
        for h in range(H):
            s0 = np.zeros((dk, v.shape[-1])) if S0 is None else f64(S0)[n, h]
            yield n, h, q[n, :, h], k[n, :, h], v[n, :, h], a[n, :, h], b[n, :, h], s0


@pytest.mark.parametrize("solve", ["corrections", "full"])
@pytest.mark.parametrize("form", [0, 1], ids=["kda", "ckda"])
@pytest.mark.parametrize("T", [64, 3 * 64 + 37])
def test_kernel_form_is_exact(form, T, solve):
    """The regrouped, block-solved chunk form equals the recurrence (fp64, no rounding)."""
    w = synth.CKDA_SPREAD.with_(B=1, T=T, H=2, dk=32, dv=24, signed_gate=form,
                                io_dtype="f32", o_dtype="f32")
    inp = synth.make_prefill(w, seed=21)
    ro, rS = oracle_prefill(inp, form)
    for n, h, q, k, v, a, b, s0 in _units(inp):
        o, S = chunk_kernel_form(q, k, v, a, b, s0, form, _Plan(tf32=False), solve)
        assert rel(o, unit_rows(ro, inp, n, h)) < 1e-11
        assert rel(S, rS[n, h]) < 1e-11


def test_block_solve_inverts_unit_lower_triangle():
    """X_i and M_ij reassemble (I + A)^{-1}: the block inverse's off-diagonal blocks are
    -sum_j M_ij (I + A)^{-1}_jk, built here row block by row block."""
    rng = np.random.default_rng(3)
    A = np.tril(rng.standard_normal((C, C)) * 0.3, -1)
    X, M = _block_solve(A, _Plan(tf32=False))
    nb = C // NB
    Tinv = np.zeros((C, C))
    for i in range(nb):
        si = slice(i * NB, (i + 1) * NB)
        Tinv[si, si] = X[i]
        for j in range(i):
            Tinv[si] -= M[(i, j)] @ Tinv[j * NB:(j + 1) * NB]
    assert np.allclose(Tinv @ (np.eye(C) + A), np.eye(C), atol=1e-10)


@pytest.mark.parametrize("solve", ["corrections", "full"])
@pytest.mark.parametrize("base,form", [(synth.KDA_STD, 0), (synth.CKDA_SPREAD, 1),
                                       (synth.KDA_STD.with_(signed_gate=1, gate="tiny"), 1)],
                         ids=["kda_std", "ckda_spread", "ckda_tiny"])
def test_tf32_operand_plan_within_tolerance(base, form, solve):
    """bf16 inputs at the full head size (d = 128, chunk 64), several chunks and a ragged
    tail: the kernel's operand plan stays at half the bf16 tolerance or below.  In the
    "tiny" CKDA case (gate logits N(0, 1.5)) the first two chunks of each head decay below
    2^-100 and take the token-by-token path, the third the factorised one."""
    w = base.with_(B=1, T=2 * 64 + 45, H=2, signed_gate=form, o_dtype="f32")
    inp = synth.make_prefill(w, seed=22)
    ro, rS = oracle_prefill(inp, form)
    os_, ss_, ro_, rs_ = [], [], [], []
    for n, h, q, k, v, a, b, s0 in _units(inp):
        o, S = chunk_kernel_form(q, k, v, a, b, s0, form, _Plan(tf32=True), solve)
        os_.append(o)
        ss_.append(S)
        ro_.append(unit_rows(ro, inp, n, h))
        rs_.append(rS[n, h])
    eo, es = rel(np.stack(os_), np.stack(ro_)), rel(np.stack(ss_), np.stack(rs_))
    assert eo < TOL_BF16 / 2 and es < TOL_BF16 / 2, (eo, es)
    # the plan rounds something: the error is far from the fp64 level
    assert eo > 1e-6 and es > 1e-6
