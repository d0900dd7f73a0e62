"""numpy front end of the fp64 CPU oracle (``ckda_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  Nothing here touches the
CUDA library, and the CUDA library never calls back into this module.

Every function takes float64 numpy arrays holding the exact values the GPU
sees (bf16 or fp32 inputs upcast to fp64) and returns float64 results.  The
recurrence and its sources are stated in the header of ``ckda_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "ckda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libckda_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_i = ctypes.c_int


def compile_c(src: str, out: str) -> str:
    """gcc -O2 a C oracle source into a shared library at ``out``."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, src,
                    "-lpthread", "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``ckda_oracle.c`` into ``_build/libckda_oracle.so`` if stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(SOURCE):
        compile_c(SOURCE, _SO)
    return _SO


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return None if x is None else x.ctypes.data_as(_dp)


class Oracle:
    """One loaded copy of the compiled oracle."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_ckda_fwd.restype = _i
        lib.oracle_ckda_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _ip,
                                        _i, _i, _i, _i, _i, _i, _i, _dp, _dp, _i]
        lib.oracle_ckda_bwd.restype = _i
        lib.oracle_ckda_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _ip,
                                        _i, _i, _i, _i, _i, _i, _i,
                                        _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _i]
        lib.oracle_decode_step.restype = _i
        lib.oracle_decode_step.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i, _i, _i, _i, _i, _dp]
        lib.oracle_transition.restype = None
        lib.oracle_transition.argtypes = [_dp, _dp, ctypes.c_double, _i, _dp]
        lib.oracle_ckda_fwd_explicit.restype = _i
        lib.oracle_ckda_fwd_explicit.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp,
                                                 _i, _i, _i, _i, _dp, _dp]
        lib.oracle_ckda_fwd_product.restype = _i
        lib.oracle_ckda_fwd_product.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _ip,
                                                _i, _i, _i, _i, _i, _i, _i, _i, _dp, _dp]
        lib.oracle_gates.restype = None
        lib.oracle_gates.argtypes = [_dp, _dp, _i, _i, _i, _dp, _dp]
        self.lib = lib

    def gates(self, a, b, signed_gate: int):
        """Activated gate alpha (shape of a) and strength beta (shape of b)."""
        a, b = _f64(a), _f64(b)
        alpha, beta = np.empty_like(a), np.empty_like(b)
        self.lib.oracle_gates(_ptr(a), _ptr(b), a.size, b.size, int(signed_gate),
                              _ptr(alpha), _ptr(beta))
        return alpha, beta

    def ckda_fwd(self, q, k, v, a, b, S0=None, cu_seqlens=None, signed_gate: int = 1,
                 threads: int = 0, want_o: bool = True):
        """Sequential fp64 forward.

        q, k, a: [B,T,H,dk]; v: [B,T,H,dv]; b: [B,T,H]; S0: [N,H,dk,dv] or None.
        With ``cu_seqlens`` (N+1 int offsets) B must be 1 and N = len(cu_seqlens)-1.
        Returns (o [B,T,H,dv] or None, S_T [N,H,dk,dv]).
        """
        q, k, v, a, b = (_f64(x) for x in (q, k, v, a, b))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        cu_p, N = None, B
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
            N = cu.size - 1
            cu_p = cu.ctypes.data_as(_ip)
        S0 = None if S0 is None else _f64(S0)
        o = np.empty((B, T, H, dv)) if want_o else None
        S_T = np.empty((N, H, dk, dv))
        rc = self.lib.oracle_ckda_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), cu_p,
                                      N, B, T, H, dk, dv, int(signed_gate), _ptr(o), _ptr(S_T),
                                      int(threads))
        if rc != 0:
            raise ValueError(f"oracle_ckda_fwd failed with code {rc}")
        return o, S_T

    def ckda_bwd(self, q, k, v, a, b, S0=None, dO=None, dS_T=None, cu_seqlens=None,
                 signed_gate: int = 1, threads: int = 0):
        """Gradients of L = sum(dO * o) + sum(dS_T * S_T) for ``ckda_fwd`` on the same
        arguments; dO [B,T,H,dv] and dS_T [N,H,dk,dv] default to zero.
        Returns (dq, dk, dv, da, db, dS0) with the shapes of q, k, v, a, b and
        [N,H,dk,dv]."""
        q, k, v, a, b = (_f64(x) for x in (q, k, v, a, b))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        cu_p, N = None, B
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
            N = cu.size - 1
            cu_p = cu.ctypes.data_as(_ip)
        S0 = None if S0 is None else _f64(S0)
        dO = None if dO is None else _f64(dO)
        dS_T = None if dS_T is None else _f64(dS_T)
        gq, gk, gv, ga = (np.empty_like(x) for x in (q, k, v, a))
        gb = np.empty_like(b)
        gS0 = np.empty((N, H, dk, dv))
        rc = self.lib.oracle_ckda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), cu_p,
                                      N, B, T, H, dk, dv, int(signed_gate), _ptr(dO), _ptr(dS_T),
                                      _ptr(gq), _ptr(gk), _ptr(gv), _ptr(ga), _ptr(gb), _ptr(gS0),
                                      int(threads))
        if rc != 0:
            raise ValueError(f"oracle_ckda_bwd failed with code {rc}")
        return gq, gk, gv, ga, gb, gS0

    def ckda_fwd_product(self, q, k, v, a, b, S0=None, cu_seqlens=None, signed_gate: int = 1):
        """DeltaProduct forward (nh rank-one updates per token, the gate once).

        q, a: [B,T,H,dk]; k: [B,T,nh,H,dk]; v: [B,T,nh,H,dv]; b: [B,T,nh,H]; S0: [N,H,dk,dv]
        or None.  Returns (o [B,T,H,dv], S_T [N,H,dk,dv])."""
        q, k, v, a, b = (_f64(x) for x in (q, k, v, a, b))
        B, T, H, dk = q.shape
        nh, dv = k.shape[2], v.shape[-1]
        cu_p, N = None, B
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
            N = cu.size - 1
            cu_p = cu.ctypes.data_as(_ip)
        S0 = None if S0 is None else _f64(S0)
        o = np.empty((B, T, H, dv))
        S_T = np.empty((N, H, dk, dv))
        rc = self.lib.oracle_ckda_fwd_product(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                              _ptr(S0), cu_p, N, B, T, H, dk, dv, nh,
                                              int(signed_gate), _ptr(o), _ptr(S_T))
        if rc != 0:
            raise ValueError(f"oracle_ckda_fwd_product failed with code {rc}")
        return o, S_T

    def decode_step(self, q, k, v, a, b, S, signed_gate: int = 1):
        """One decode step.  Returns (o [B,H,dv], S_new [B,H,dk,dv]); S is not modified."""
        q, k, v, a, b = (_f64(x) for x in (q, k, v, a, b))
        S = _f64(S).copy()
        B, H, dk = q.shape
        dv = v.shape[-1]
        o = np.empty((B, H, dv))
        rc = self.lib.oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S),
                                         B, H, dk, dv, int(signed_gate), _ptr(o))
        if rc != 0:
            raise ValueError(f"oracle_decode_step failed with code {rc}")
        return o, S

    def transition(self, k, alpha, beta: float):
        """Dense A = (I - beta k k^T) Diag(alpha)."""
        k, alpha = _f64(k), _f64(alpha)
        n = k.size
        A = np.empty((n, n))
        self.lib.oracle_transition(_ptr(k), _ptr(alpha), float(beta), n, _ptr(A))
        return A

    def ckda_fwd_explicit(self, q, k, v, a, b, S0=None, signed_gate: int = 1):
        """Explicit-matrix forward, one sequence and head: q,k,a [T,dk], v [T,dv], b [T]."""
        q, k, v, a, b = (_f64(x) for x in (q, k, v, a, b))
        T, dk = q.shape
        dv = v.shape[-1]
        S0 = None if S0 is None else _f64(S0)
        o = np.empty((T, dv))
        S_T = np.empty((dk, dv))
        rc = self.lib.oracle_ckda_fwd_explicit(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                               _ptr(S0), T, dk, dv, int(signed_gate),
                                               _ptr(o), _ptr(S_T))
        if rc != 0:
            raise ValueError(f"oracle_ckda_fwd_explicit failed with code {rc}")
        return o, S_T


_lock = threading.Lock()
_default = None


def default() -> Oracle:
    """The oracle built from ``ckda_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def gates(*a, **kw):
    return default().gates(*a, **kw)


def ckda_fwd(*a, **kw):
    return default().ckda_fwd(*a, **kw)


def ckda_bwd(*a, **kw):
    return default().ckda_bwd(*a, **kw)


def decode_step(*a, **kw):
    return default().decode_step(*a, **kw)


def ckda_fwd_product(*a, **kw):
    return default().ckda_fwd_product(*a, **kw)


def transition(*a, **kw):
    return default().transition(*a, **kw)


def ckda_fwd_explicit(*a, **kw):
    return default().ckda_fwd_explicit(*a, **kw)
