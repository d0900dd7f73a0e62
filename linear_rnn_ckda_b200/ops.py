"""Python binding of ``libckda.so`` (the C ABI in ``include/ckda.h``).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the recurrence runs in the library's kernels.
There is no CPU fallback: if the library is missing or the tensors are not on
a CUDA device, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libckda.so")
_lock = threading.Lock()
_lib = None

CKDA_F32 = 0
CKDA_BF16 = 1
# flags OR-ed into signed_gate (include/ckda.h)
GATE_PER_HEAD = 16   # one gate logit per token and head: a is [B,T,H] ([B,H] for decode)
QK_L2NORM = 32       # q and k are L2-normalised inside the kernels
DELTA_PRODUCT2 = 64  # two keys, values, strengths per token: k [B,T,2,H,dk], v [B,T,2,H,dv], b [B,T,2,H]
_DT = {torch.float32: CKDA_F32, torch.bfloat16: CKDA_BF16}
_TORCH_DT = {CKDA_F32: torch.float32, CKDA_BF16: torch.bfloat16}

_vp = ctypes.c_void_p
_i = ctypes.c_int

# name -> (restype, argtypes), mirroring include/ckda.h
SIGNATURES = {
    "ckda_chunk_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                            _i, _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "ckda_chunk_fwd_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i]),
    "ckda_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]),
    "ckda_chunk_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                            _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                            _vp]),
    "ckda_chunk_bwd_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i]),
    "ckda_chunk_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _i, _i, _vp, _vp, _vp]),
    "ckda_workspace_status": (_i, [_vp, ctypes.POINTER(_i), _vp]),
    "ckda_noalloc_status": (_i, [ctypes.POINTER(_i), _vp]),
    "ckda_debug_wait_injection": (None, [_i, ctypes.c_ulonglong]),
    "ckda_debug_segment_split": (None, [_i, _i]),
    "ckda_debug_segment_choice": (_i, [ctypes.POINTER(ctypes.c_int32), _i, _i, _i,
                                      ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "ckda_status_string": (ctypes.c_char_p, [_i]),
    "ckda_version": (_i, []),
}


class CkdaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} (code {code})")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def load():
    """Loads ``libckda.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with `python -m linear_rnn_ckda_b200.build` "
                    "(there is no CPU fallback)")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().ckda_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _same_device(ref: torch.Tensor, **tensors):
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, q on {ref.device}")


def check_prefill_args(q, k, v, a, b, S0=None, cu_seqlens=None, o=None, S_T=None,
                       o_dtype=None, signed_gate: int = 0):
    """Shapes, dtypes and devices that ``ckda_chunk_fwd`` relies on but cannot see (it receives
    bare pointers, so a short or mistyped buffer would be read or written past its end).
    Raises ValueError; returns (N, dv).  The offsets inside ``cu_seqlens`` are checked on the
    device (the workspace status word), not here."""
    _need(q.dim() == 4, f"q must be [B,T,H,dk], got {tuple(q.shape)}")
    _need(q.dtype in _DT, f"q must be float32 or bfloat16, got {q.dtype}")
    B, T, H, dk = q.shape
    p2 = bool(signed_gate & DELTA_PRODUCT2)
    lead = (B, T, 2, H) if p2 else (B, T, H)   # rows of k, v, b (two per token for DeltaProduct2)
    _need(tuple(k.shape) == lead + (dk,) and k.dtype == q.dtype,
          f"k must be {lead + (dk,)} in q's dtype, got {tuple(k.shape)}, {k.dtype}")
    a_shape = (B, T, H) if signed_gate & GATE_PER_HEAD else tuple(q.shape)
    _need(tuple(a.shape) == a_shape and a.dtype == q.dtype,
          f"a must be {a_shape} in q's dtype, got {tuple(a.shape)}, {a.dtype}")
    _need(v.dim() == len(lead) + 1 and tuple(v.shape[:-1]) == lead and v.dtype == q.dtype,
          f"v must be {lead + ('dv',)} in q's dtype, got {tuple(v.shape)}, {v.dtype}")
    dv = v.shape[-1]
    _need(tuple(b.shape) == lead and b.dtype == torch.float32,
          f"b must be {lead} float32, got {tuple(b.shape)}, {b.dtype}")
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1 and cu_seqlens.dtype == torch.int32,
              "cu_seqlens must be a 1-D int32 tensor of N+1 offsets")
        _need(B == 1, "packed sequences (cu_seqlens) need B == 1")
        N = cu_seqlens.numel() - 1
    for name, t in (("S0", S0), ("S_T", S_T)):
        _need(t is None or (t.shape == (N, H, dk, dv) and t.dtype == torch.float32),
              f"{name} must be [N,H,dk,dv] = {(N, H, dk, dv)} float32")
    od = q.dtype if o_dtype is None else o_dtype
    _need(od in _DT, f"o_dtype must be float32 or bfloat16, got {od}")
    _need(o is None or (o.shape == (B, T, H, dv) and o.dtype == od),
          f"o must be [B,T,H,dv] = {(B, T, H, dv)} in {od}")
    _same_device(q, k=k, v=v, a=a, b=b, S0=S0, cu_seqlens=cu_seqlens, o=o, S_T=S_T)
    return N, dv


def check_decode_args(q, k, v, a, b, S, o=None, o_dtype=None, signed_gate: int = 0):
    """The same checks for ``ckda_decode_step``: q, k, a [B,H,dk]; v [B,H,dv] in q's dtype;
    b [B,H] float32; S [B,H,dk,dv] float32; o [B,H,dv] in the output dtype."""
    _need(q.dim() == 3, f"q must be [B,H,dk], got {tuple(q.shape)}")
    _need(q.dtype in _DT, f"q must be float32 or bfloat16, got {q.dtype}")
    B, H, dk = q.shape
    lead = (B, 2, H) if signed_gate & DELTA_PRODUCT2 else (B, H)
    _need(tuple(k.shape) == lead + (dk,) and k.dtype == q.dtype,
          f"k must be {lead + (dk,)} in q's dtype, got {tuple(k.shape)}, {k.dtype}")
    a_shape = (B, H) if signed_gate & GATE_PER_HEAD else tuple(q.shape)
    _need(tuple(a.shape) == a_shape and a.dtype == q.dtype,
          f"a must be {a_shape} in q's dtype, got {tuple(a.shape)}, {a.dtype}")
    _need(v.dim() == len(lead) + 1 and tuple(v.shape[:-1]) == lead and v.dtype == q.dtype,
          f"v must be {lead + ('dv',)} in q's dtype, got {tuple(v.shape)}, {v.dtype}")
    dv = v.shape[-1]
    _need(tuple(b.shape) == lead and b.dtype == torch.float32,
          f"b must be {lead} float32, got {tuple(b.shape)}, {b.dtype}")
    _need(S.shape == (B, H, dk, dv) and S.dtype == torch.float32,
          f"S must be [B,H,dk,dv] = {(B, H, dk, dv)} float32")
    od = q.dtype if o_dtype is None else o_dtype
    _need(od in _DT, f"o_dtype must be float32 or bfloat16, got {od}")
    _need(o is None or (o.shape == (B, H, dv) and o.dtype == od),
          f"o must be [B,H,dv] = {(B, H, dv)} in {od}")
    _same_device(q, k=k, v=v, a=a, b=b, S=S, o=o)
    return dv


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def workspace_size(B, T, H, dk, dv, chunk, n_seqs=0) -> int:
    return int(load().ckda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, n_seqs))


def new_workspace(B, T, H, dk, dv, chunk, n_seqs=0, device=None) -> torch.Tensor:
    n = workspace_size(B, T, H, dk, dv, chunk, n_seqs)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def chunk_fwd(q, k, v, a, b, S0=None, cu_seqlens=None, chunk: int = 64, signed_gate: int = 1,
              o_dtype=None, o=None, S_T=None, workspace=None, want_o: bool = True,
              want_state: bool = True):
    """Chunkwise forward.  Returns (o, S_T) (either may be None when not wanted).

    q, k, a: [B,T,H,dk]; v: [B,T,H,dv] (fp32 or bf16, same dtype); b: [B,T,H] fp32;
    S0: [N,H,dk,dv] fp32 or None; cu_seqlens: int32 CUDA tensor [N+1] or None.
    """
    lib = load()
    N, dv = check_prefill_args(q, k, v, a, b, S0, cu_seqlens, o, S_T, o_dtype, signed_gate)
    B, T, H, dk = q.shape
    io = _DT[q.dtype]
    od = io if o_dtype is None else _DT[o_dtype]
    dev = q.device
    if want_o and o is None:
        o = torch.empty((B, T, H, dv), dtype=_TORCH_DT[od], device=dev)
    if want_state and S_T is None:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(B, T, H, dk, dv, chunk, N if cu_seqlens is not None else 0, dev)
    _need(workspace.device == dev, f"workspace is on {workspace.device}, q on {dev}")
    rc = lib.ckda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0),
                            _ptr(cu_seqlens), N if cu_seqlens is not None else 0, B, T, H, dk, dv,
                            chunk, signed_gate, io, od, _ptr(o if want_o else None),
                            _ptr(S_T if want_state else None), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(dev))
    if rc != 0:
        raise CkdaError("ckda_chunk_fwd", rc)
    return (o if want_o else None), (S_T if want_state else None)


def bwd_workspace_size(B, T, H, dk, dv, n_seqs=0) -> int:
    return int(load().ckda_chunk_bwd_workspace_size(B, T, H, dk, dv, n_seqs))


def chunk_bwd(q, k, v, a, b, S0=None, cu_seqlens=None, dO=None, dS_T=None,
              signed_gate: int = 1, want_dS0: bool = True, workspace=None, grads=None):
    """Backward of ``chunk_fwd``: gradients of sum(dO * o) + sum(dS_T * S_T).

    Returns (dq, dk, dv, da, db, dS0) as float32 tensors with the shapes of q, k, v, a, b and
    S0's [N,H,dk,dv] (dS0 None when not wanted).  dO: [B,T,H,dv] float32 or bfloat16, or None
    (zero); dS_T: [N,H,dk,dv] float32 or None (zero).  ``grads`` may supply the six output
    tensors."""
    lib = load()
    N, dv = check_prefill_args(q, k, v, a, b, S0, cu_seqlens, signed_gate=signed_gate)
    B, T, H, dk = q.shape
    dev = q.device
    _need(dO is None or (dO.shape == (B, T, H, dv) and dO.dtype in _DT),
          f"dO must be [B,T,H,dv] = {(B, T, H, dv)} float32 or bfloat16")
    _need(dS_T is None or (dS_T.shape == (N, H, dk, dv) and dS_T.dtype == torch.float32),
          f"dS_T must be [N,H,dk,dv] = {(N, H, dk, dv)} float32")
    _same_device(q, dO=dO, dS_T=dS_T)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = (torch.empty((B, T, H, dk), **f32), torch.empty((B, T, H, dk), **f32),
                 torch.empty((B, T, H, dv), **f32), torch.empty(tuple(a.shape), **f32),
                 torch.empty((B, T, H), **f32),
                 torch.empty((N, H, dk, dv), **f32) if want_dS0 else None)
    gq, gk, gv, ga, gb, gS0 = grads
    for name, t, shape in (("dq", gq, (B, T, H, dk)), ("dk", gk, (B, T, H, dk)),
                           ("dv", gv, (B, T, H, dv)), ("da", ga, tuple(a.shape)),
                           ("db", gb, (B, T, H)), ("dS0", gS0, (N, H, dk, dv))):
        _need(t is None or (tuple(t.shape) == shape and t.dtype == torch.float32),
              f"{name} must be {shape} float32")
    _need(gS0 is not None or not want_dS0, "dS0 buffer missing")
    n = bwd_workspace_size(B, T, H, dk, dv, N if cu_seqlens is not None else 0)
    if workspace is None:
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    rc = lib.ckda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S0), _ptr(cu_seqlens),
                            N if cu_seqlens is not None else 0, B, T, H, dk, dv, signed_gate,
                            _DT[q.dtype], _ptr(dO), _DT[dO.dtype] if dO is not None else CKDA_F32,
                            _ptr(dS_T), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(ga), _ptr(gb),
                            _ptr(gS0), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(dev))
    if rc != 0:
        raise CkdaError("ckda_chunk_bwd", rc)
    return gq, gk, gv, ga, gb, gS0


def decode_step(q, k, v, a, b, S, signed_gate: int = 1, o_dtype=None, o=None, want_o=True):
    """One decode step; S [B,H,dk,dv] fp32 is updated in place.  Returns o [B,H,dv]."""
    lib = load()
    dv = check_decode_args(q, k, v, a, b, S, o, o_dtype, signed_gate)
    B, H, dk = q.shape
    io = _DT[q.dtype]
    od = io if o_dtype is None else _DT[o_dtype]
    if want_o and o is None:
        o = torch.empty((B, H, dv), dtype=_TORCH_DT[od], device=q.device)
    rc = lib.ckda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S), B, H, dk, dv,
                              signed_gate, io, od, _ptr(o if want_o else None), _stream(q.device))
    if rc != 0:
        raise CkdaError("ckda_decode_step", rc)
    return o if want_o else None


def noalloc_status(device=None) -> int:
    """Device status word of the last ``ckda_chunk_fwd_noalloc`` call on the current device
    (synchronises the current stream)."""
    st = ctypes.c_int(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    rc = load().ckda_noalloc_status(ctypes.byref(st), _stream(dev))
    if rc != 0:
        raise CkdaError("ckda_noalloc_status", rc)
    return st.value


def debug_wait_injection(chunk_index: int, wait_ns: int = 0) -> None:
    """Test hook: see ``ckda_debug_wait_injection`` in ``include/ckda.h`` (-1 switches it off)."""
    load().ckda_debug_wait_injection(int(chunk_index), int(wait_ns))


def debug_segment_choice(lengths, H: int, sm_count: int = 148):
    """Test hook: see ``ckda_debug_segment_choice`` in ``include/ckda.h``.  Returns
    (sequences cut, [segments of each])."""
    n = len(lengths)
    arr = (ctypes.c_int32 * max(n, 1))(*[int(x) for x in lengths])
    k = ctypes.c_int(0)
    m = (ctypes.c_int * 2)()
    rc = load().ckda_debug_segment_choice(arr, n, int(H), int(sm_count), ctypes.byref(k), m)
    if rc != 0:
        raise CkdaError("ckda_debug_segment_choice", rc)
    return k.value, [m[i] for i in range(k.value)]


def debug_segment_split(n_split: int, n_segments: int) -> None:
    """Test hook: see ``ckda_debug_segment_split`` in ``include/ckda.h`` (0, 0 switches it off)."""
    load().ckda_debug_segment_split(int(n_split), int(n_segments))


def workspace_status(workspace: torch.Tensor) -> int:
    """Device status word of the last chunk_fwd that used ``workspace`` (synchronises)."""
    st = ctypes.c_int(0)
    rc = load().ckda_workspace_status(_ptr(workspace), ctypes.byref(st), _stream(workspace.device))
    if rc != 0:
        raise CkdaError("ckda_workspace_status", rc)
    return st.value
