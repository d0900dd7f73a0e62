"""Seeded synthetic inputs shaped like the Complex-KDA review's workloads.

This module draws random numbers and nothing else: it holds none of the
recurrence's arithmetic, so both the CUDA path and the CPU oracle can consume
what it produces.  Values are drawn in float64 with numpy's PCG64 generator,
one independent stream per tensor (``SeedSequence([seed, stream])``), q and k
are L2-normalised per (token, head) in float64, and everything is rounded once
(round-to-nearest-even) to the io dtype with torch on the host.

Distributions (N(mu, s): s is the standard deviation):
  * q, k ~ N(0,1) then L2-normalised per token and head; v ~ N(0,1)
  * gate logits a, per (token, head, channel):
      "std"     N(4, 1)                    (KDA, gates near 1)
      "tiny"    N(0, 1.5)                  (about half of CKDA gates negative)
      "spread"  0.5 N(3,1) + 0.5 N(-3,1)   (spread initialisation, fair coin)
      "fast"    N(-2, 1) on every fourth key channel (c % 4 == 0), N(4, 1) on the others
                (fast-forgetting channels beside slow ones)
  * strength logits b, per (token, head):
      "std"     N(0, 1)
      "spread"  0.5 N(-2,0.5) + 0.5 N(2,0.5)
  * initial state S0 ~ N(0, 0.02) per entry, or zero.
The spread initialisation and the bimodal strength come from the CKDA review
("Method steps", step 1); the head shape dk = dv = 128 and 16 heads follow
its throughput figure (Figure 5).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np
import torch

# stream ids (fixed so that every tensor has its own reproducible sub-stream)
_S_Q, _S_K, _S_V, _S_A, _S_B, _S_S0, _S_LEN, _S_ACOIN, _S_BCOIN = range(1, 10)

_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic workload."""
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    signed_gate: int          # 0 KDA, 1 CKDA
    gate: str                 # "std" | "tiny" | "spread"
    strength: str             # "std" | "spread"
    s0: bool                  # draw S0 ~ N(0,0.02) (else zero / None)
    io_dtype: str = "bf16"
    o_dtype: str = "bf16"
    seq_lens: Optional[tuple] = None   # packed varlen (B must be 1), or None
    decode_steps: int = 0     # >0: a decode workload of this many steps (T unused)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return sum(self.seq_lens) if self.seq_lens is not None else self.B * self.T

    @property
    def n_seqs(self) -> int:
        return len(self.seq_lens) if self.seq_lens is not None else self.B


def varlen_lengths(seed: int = 0, n_short: int = 16, lo: int = 512, hi: int = 8192,
                   long_len: int = 65536) -> tuple:
    """16 lengths uniform on {512..8192} (inclusive) followed by one of 65,536."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, _S_LEN]))
    short = rng.integers(lo, hi + 1, size=n_short)
    return tuple(int(x) for x in short) + (int(long_len),)


# The five workloads.  Names state what they are and their sizes.
TINY_CKDA_FP32 = Workload("tiny_ckda_fp32_b1_t64_h1_d16_c16", 1, 64, 1, 16, 16, 16, 1,
                          "tiny", "std", False, io_dtype="f32", o_dtype="f32")
KDA_STD = Workload("kda_std_b4_t4096_h16_d128_c64", 4, 4096, 16, 128, 128, 64, 0,
                   "std", "std", False)
CKDA_SPREAD = Workload("ckda_spread_b8_t8192_h16_d128_c64", 8, 8192, 16, 128, 128, 64, 1,
                       "spread", "spread", True)
CKDA_VARLEN = Workload("ckda_varlen_h32_16x[512,8192]+65536_d128_c64", 1, 0, 32, 128, 128, 64, 1,
                       "spread", "spread", True, seq_lens=None)
# KDA with a quarter of the key channels forgetting fast (a robustness workload, not one of the
# pages' configurations)
KDA_FAST = Workload("kda_fastforget_b4_t4096_h16_d128_c64", 4, 4096, 16, 128, 128, 64, 0,
                    "fast", "std", False)
DECODE = Workload("ckda_decode_b256_h32_d128_128steps", 256, 1, 32, 128, 128, 64, 1,
                  "spread", "spread", True, io_dtype="bf16", o_dtype="f32", decode_steps=128)


def varlen_workload(seed: int = 0) -> Workload:
    lens = varlen_lengths(seed)
    return CKDA_VARLEN.with_(seq_lens=lens, T=sum(lens))


def _rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, stream, sub]))


def _to_torch(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(x).to(_DTYPES[dtype])


def _normal_slabs(rng, shape, mu, sd, dtype, l2_last=False, slab=1 << 23):
    """Draw N(mu, sd) of ``shape`` in float64 slabs and round to ``dtype``."""
    out = torch.empty(shape, dtype=_DTYPES[dtype])
    flat = out.view(-1, shape[-1])
    rows = flat.shape[0]
    step = max(1, slab // shape[-1])
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = rng.normal(mu, sd, size=(r1 - r0, shape[-1]))
        if l2_last:
            x /= np.linalg.norm(x, axis=-1, keepdims=True)
        flat[r0:r1] = _to_torch(x, dtype)
    return out


def _mixture_slabs(rng_v, rng_c, shape, comps, dtype, slab=1 << 23):
    """Fair-coin mixture of normals ``comps`` = ((mu0, sd0), (mu1, sd1))."""
    out = torch.empty(shape, dtype=_DTYPES[dtype])
    flat = out.view(-1)
    n = flat.numel()
    for i0 in range(0, n, slab):
        i1 = min(n, i0 + slab)
        coin = rng_c.integers(0, 2, size=i1 - i0)
        z = rng_v.standard_normal(size=i1 - i0)
        mu = np.where(coin == 0, comps[0][0], comps[1][0])
        sd = np.where(coin == 0, comps[0][1], comps[1][1])
        flat[i0:i1] = _to_torch(mu + sd * z, dtype)
    return out


def _gate_logits(w: Workload, shape, seed: int, sub: int = 0):
    if w.gate == "std":
        return _normal_slabs(_rng(seed, _S_A, sub), shape, 4.0, 1.0, w.io_dtype)
    if w.gate == "tiny":
        return _normal_slabs(_rng(seed, _S_A, sub), shape, 0.0, 1.5, w.io_dtype)
    if w.gate == "spread":
        return _mixture_slabs(_rng(seed, _S_A, sub), _rng(seed, _S_ACOIN, sub), shape,
                              ((3.0, 1.0), (-3.0, 1.0)), w.io_dtype)
    if w.gate == "fast":
        out = _normal_slabs(_rng(seed, _S_A, sub), shape, 0.0, 1.0, "f32")   # z ~ N(0, 1)
        mu = torch.full((shape[-1],), 4.0)
        mu[0::4] = -2.0
        return (out + mu).to(_DTYPES[w.io_dtype])
    raise ValueError(w.gate)


def _strength_logits(w: Workload, shape, seed: int, sub: int = 0):
    if w.strength == "std":
        return _normal_slabs(_rng(seed, _S_B, sub), shape, 0.0, 1.0, "f32")
    if w.strength == "spread":
        return _mixture_slabs(_rng(seed, _S_B, sub), _rng(seed, _S_BCOIN, sub), shape,
                              ((-2.0, 0.5), (2.0, 0.5)), "f32")
    raise ValueError(w.strength)


def make_prefill(w: Workload, seed: int = 0) -> dict:
    """Host (CPU) tensors for one forward call of workload ``w``.

    Returns q, k, a [B,T,H,dk] and v [B,T,H,dv] in the io dtype, b [B,T,H]
    float32, S0 [N,H,dk,dv] float32 or None, cu_seqlens int32 [N+1] or None.
    """
    if w.seq_lens is not None:
        B, T = 1, sum(w.seq_lens)
    else:
        B, T = w.B, w.T
    H, dk, dv = w.H, w.dk, w.dv
    out = {
        "q": _normal_slabs(_rng(seed, _S_Q), (B, T, H, dk), 0.0, 1.0, w.io_dtype, l2_last=True),
        "k": _normal_slabs(_rng(seed, _S_K), (B, T, H, dk), 0.0, 1.0, w.io_dtype, l2_last=True),
        "v": _normal_slabs(_rng(seed, _S_V), (B, T, H, dv), 0.0, 1.0, w.io_dtype),
        "a": _gate_logits(w, (B, T, H, dk), seed),
        "b": _strength_logits(w, (B, T, H), seed),
    }
    N = w.n_seqs
    out["S0"] = (_normal_slabs(_rng(seed, _S_S0), (N, H, dk, dv), 0.0, 0.02, "f32")
                 if w.s0 else None)
    if w.seq_lens is not None:
        cu = np.zeros(len(w.seq_lens) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(np.asarray(w.seq_lens, dtype=np.int64))
        out["cu_seqlens"] = torch.from_numpy(cu)
    else:
        out["cu_seqlens"] = None
    return out


def make_decode(w: Workload, seed: int = 0, steps: Optional[int] = None) -> dict:
    """Host tensors for ``steps`` successive decode steps of workload ``w``.

    q, k, a [steps,B,H,dk], v [steps,B,H,dv] in the io dtype; b [steps,B,H]
    float32; S [B,H,dk,dv] float32 ~ N(0, 0.02) (or zeros).
    """
    steps = w.decode_steps if steps is None else steps
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    out = {
        "q": _normal_slabs(_rng(seed, _S_Q), (steps, B, H, dk), 0.0, 1.0, w.io_dtype, l2_last=True),
        "k": _normal_slabs(_rng(seed, _S_K), (steps, B, H, dk), 0.0, 1.0, w.io_dtype, l2_last=True),
        "v": _normal_slabs(_rng(seed, _S_V), (steps, B, H, dv), 0.0, 1.0, w.io_dtype),
        "a": _gate_logits(w, (steps, B, H, dk), seed),
        "b": _strength_logits(w, (steps, B, H), seed),
    }
    out["S"] = (_normal_slabs(_rng(seed, _S_S0), (B, H, dk, dv), 0.0, 0.02, "f32")
                if w.s0 else torch.zeros((B, H, dk, dv), dtype=torch.float32))
    return out
