"""Shared helpers of the parity tests: run the CUDA path and the oracle on the
same seeded inputs and measure relative Frobenius errors."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances (relative Frobenius error on o and on the final state):
TOL_FP32 = 1e-5      # fp32 q/k/v/a and o
TOL_BF16 = 2e-3      # bf16 q/k/v/a, fp32 state and accumulation


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def rel(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    d = np.linalg.norm(x - ref)
    return float(d / n) if n > 0 else float(d)


# The row guard's factor on the global bar.  Row errors spread around the global figure
# (a row whose norm is small next to the state it reads has a larger relative error); twice
# the bar still fails a single wrong element of typical size by more than an order of
# magnitude (one such element in a 128-wide row is a relative error near 1/sqrt(128)).
ROW_FACTOR = 2.0

# Half a unit in the last place of a bf16 value, relative to the value: bf16 keeps 8
# significant bits, so round-to-nearest moves a value by at most 2^-8 of its magnitude.
BF16_HALF_ULP = 2.0 ** -8


def row_errors(x, ref):
    """Per-row (last axis) error figures: relative 2-norm error of each row, the largest
    absolute error of each row, and the reference's largest magnitude."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = x.reshape(-1, x.shape[-1]) - ref.reshape(-1, ref.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    en = np.linalg.norm(d, axis=1)
    rn = np.linalg.norm(r, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        rel_rows = np.where(rn > 0, en / np.where(rn > 0, rn, 1.0), en)
    return rel_rows, np.abs(d).max(axis=1) if d.size else np.zeros(0), float(np.abs(r).max(initial=0.0))


def assert_close(x, ref, tol, what="", bf16_out=False):
    """The parity bar of the GPU tests, on one output tensor.

    x: the CUDA path's result; ref: the oracle's fp64 result (NOT rounded); rows are the last
    axis (one token-head row of o, one key-channel row of a state).

    - Global: relative Frobenius error <= tol, against the oracle rounded to bf16 when the
      output is bf16 (round-to-nearest-even, as the kernels store it).
    - Every row: relative error <= ROW_FACTOR * tol, or largest absolute error
      <= ROW_FACTOR * tol * max|ref| (a row whose own norm is small next to the rest is judged
      on the tensor's scale).  For a bf16 output each element must lie within its rounding
      bound, 2^-8 |ref|, plus tol * max|ref| of the unrounded oracle.
    A single wrong element of typical size fails the row test even when it moves the global
    figure by less than tol.  Returns (global error, worst row figure) for reports.
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (what, x.shape, ref.shape)
    assert np.all(np.isfinite(x)), (what, "non-finite values")
    gref = bf16_round(ref) if bf16_out else ref
    g = rel(x, gref)
    assert g <= tol, (what, "global relative error", g, tol)
    if x.size == 0:
        return g, 0.0
    scale = float(np.abs(ref).max(initial=0.0))
    if bf16_out:
        bound = BF16_HALF_ULP * np.abs(ref) + tol * scale
        excess = np.abs(x - ref) - bound
        worst = float(excess.max())
        assert worst <= 0.0, (what, "element outside bf16 rounding + tol", worst,
                              np.unravel_index(int(np.argmax(excess)), x.shape))
        return g, worst
    rel_rows, max_rows, scale = row_errors(x, ref)
    rt = ROW_FACTOR * tol
    ok = (rel_rows <= rt) | (max_rows <= rt * scale)
    if not np.all(ok):
        bad = int(np.argmin(ok))
        raise AssertionError((what, "row error", int(bad), float(rel_rows[bad]),
                              float(max_rows[bad]), tol, scale))
    return g, float(np.minimum(rel_rows, max_rows / max(scale, 1e-300)).max())


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to bf16 (torch on the host), back to float64."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def to_device(inp: dict, device="cuda") -> dict:
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}


def oracle_prefill(inp: dict, signed_gate: int, threads: int = 0):
    """Oracle forward on host inputs (upcast to fp64)."""
    cu = None if inp.get("cu_seqlens") is None else inp["cu_seqlens"].numpy()
    return oracle.ckda_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["a"]), f64(inp["b"]),
                           f64(inp.get("S0")), cu_seqlens=cu, signed_gate=signed_gate,
                           threads=threads)


def unit_rows(o: np.ndarray, inp: dict, n: int, h: int) -> np.ndarray:
    cu = inp.get("cu_seqlens")
    if cu is not None:
        return o[0, int(cu[n]):int(cu[n + 1]), h, :]
    return o[n, :, h, :]


def _segments(inp: dict):
    """(sequence index, batch row, t0, t1) of every sequence of a forward's inputs."""
    cu = inp.get("cu_seqlens")
    B, T = inp["q"].shape[:2]
    if cu is None:
        return [(n, n, 0, T) for n in range(B)]
    cu = [int(x) for x in cu]
    return [(n, 0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def compare_prefill_whole(o, S, inp: dict, signed_gate: int, tol: float, bf16_out: bool = False,
                          block: int = 1 << 19, threads: int = 0):
    """Whole-tensor parity of a forward's outputs (host or device tensors o [B,T,H,dv] and
    S_T [N,H,dk,dv]) against the oracle on the same inputs, every sequence and head.

    The oracle runs on blocks of one sequence and up to ``block`` token-heads, so host memory
    stays bounded on the largest workloads; assert_close's global and row bars hold on every
    block, hence on the whole tensors.  Returns the worst block's (o, S) global errors."""
    q, k, v, a, b = (inp[x] for x in "qkvab")
    S0 = inp.get("S0")
    H = q.shape[2]
    o = o.detach().cpu() if isinstance(o, torch.Tensor) else o
    S = S.detach().cpu() if isinstance(S, torch.Tensor) else S
    worst = [0.0, 0.0]
    for (n, row, t0, t1) in _segments(inp):
        L = t1 - t0
        hb = max(1, min(H, block // max(L, 1)))
        for h0 in range(0, H, hb):
            h1 = min(H, h0 + hb)
            sl = (slice(row, row + 1), slice(t0, t1), slice(h0, h1))
            s0 = None if S0 is None else f64(S0[n:n + 1, h0:h1])
            ro, rS = oracle.ckda_fwd(f64(q[sl]), f64(k[sl]), f64(v[sl]), f64(a[sl]), f64(b[sl]),
                                     s0, signed_gate=signed_gate, threads=threads)
            tag = f"seq {n} heads {h0}..{h1 - 1}"
            if L > 0:
                eo, _ = assert_close(f64(o[sl]), ro, tol, "o " + tag, bf16_out=bf16_out)
                worst[0] = max(worst[0], eo)
            es, _ = assert_close(f64(S[n:n + 1, h0:h1]), rS, tol, "S_T " + tag)
            worst[1] = max(worst[1], es)
    return tuple(worst)


GRAD_NAMES = ("dq", "dk", "dv", "da", "db", "dS0")


def compare_bwd_whole(grads, inp: dict, dO, dS_T, signed_gate: int, tol: float,
                      block: int = 1 << 18, threads: int = 0):
    """Whole-tensor parity of the backward's six gradients (host or device tensors) against
    the oracle's backward on the same inputs, sequence by sequence and in head blocks of at
    most ``block`` token-heads (host memory stays bounded).  assert_close's bars hold on
    every block.  Returns the worst block's global error per gradient."""
    q, k, v, a, b = (inp[x] for x in "qkvab")
    S0 = inp.get("S0")
    H = q.shape[2]
    grads = [None if g is None else g.detach().cpu() for g in grads]
    dO = None if dO is None else dO.detach().cpu()
    dS_T = None if dS_T is None else dS_T.detach().cpu()
    worst = dict.fromkeys(GRAD_NAMES, 0.0)
    for (n, row, t0, t1) in _segments(inp):
        L = t1 - t0
        hb = max(1, min(H, block // max(L, 1)))
        for h0 in range(0, H, hb):
            h1 = min(H, h0 + hb)
            sl = (slice(row, row + 1), slice(t0, t1), slice(h0, h1))
            ss = (slice(n, n + 1), slice(h0, h1))
            ref = oracle.ckda_bwd(f64(q[sl]), f64(k[sl]), f64(v[sl]), f64(a[sl]), f64(b[sl]),
                                  None if S0 is None else f64(S0[ss]),
                                  dO=None if dO is None else f64(dO[sl]),
                                  dS_T=None if dS_T is None else f64(dS_T[ss]),
                                  signed_gate=signed_gate, threads=threads)
            tag = f"seq {n} heads {h0}..{h1 - 1}"
            for i, name in enumerate(GRAD_NAMES):
                g = grads[i]
                if g is None:
                    continue
                got = f64(g[ss]) if name == "dS0" else f64(g[sl])
                if got.size == 0:
                    continue
                e, _ = assert_close(got, ref[i], tol, f"{name} {tag}")
                worst[name] = max(worst[name], e)
    return worst
