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


def oracle_units(inp: dict, signed_gate: int, units, threads: int = 0):
    """Oracle forward restricted to (sequence, head) units.

    Returns {(n, h): (o_rows [len, dv], S_T [dk, dv])}; the rows are the
    unit's tokens in order.
    """
    q, k, v, a, b = (inp[x] for x in "qkvab")
    S0 = inp.get("S0")
    cu = inp.get("cu_seqlens")
    out = {}
    for (n, h) in units:
        if cu is not None:
            t0, t1 = int(cu[n]), int(cu[n + 1])
            sl = (slice(0, 1), slice(t0, t1), slice(h, h + 1))
        else:
            sl = (slice(n, n + 1), slice(None), slice(h, h + 1))
        s0 = None if S0 is None else f64(S0[n:n + 1, h:h + 1])
        o, S = oracle.ckda_fwd(f64(q[sl]), f64(k[sl]), f64(v[sl]), f64(a[sl]), f64(b[sl]), s0,
                               signed_gate=signed_gate, threads=threads)
        out[(n, h)] = (o[0, :, 0, :], S[0, 0])
    return out


def unit_rows(o: np.ndarray, inp: dict, n: int, h: int) -> np.ndarray:
    cu = inp.get("cu_seqlens")
    if cu is not None:
        return o[0, int(cu[n]):int(cu[n + 1]), h, :]
    return o[n, :, h, :]
