"""The per-head (GDN-style scalar) gate and the in-kernel q/k L2 normalisation on every
kernel (exact and tensor-core forward, decode, backward), against the oracle fed the plain
definitions: the per-head gate broadcast over the key channels (a scalar gate is a
channel-wise gate whose channels are equal; CKDA review, "Scalar vs channel-wise gating"),
and q, k divided by their norms in fp64 on the host (the fused normalisation of the review's
"Reproducibility" section).  For the backward, the oracle's gradients with respect to the
normalised q, k are carried through the normalisation, dy = (dx - x (x . dx)) / ||y||, and
the per-head gate's gradient is the sum of the channel gradients."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL_BF16, TOL_FP32, assert_close, f64, to_device
from linear_rnn_ckda_b200 import ops as ops_mod
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu
PH, L2 = ops_mod.GATE_PER_HEAD, ops_mod.QK_L2NORM
TOL_BWD = 1e-4


def _raw_inputs(w, seed, flags):
    """Inputs for the flagged call: per-head logits [B,T,H] (first channel's draws), and q, k
    of random norms (one row of each set to zero) when normalising in the kernel."""
    inp = synth.make_prefill(w, seed)
    dt = inp["q"].dtype
    if flags & PH:
        inp["a"] = inp["a"][..., 0].contiguous()
    if flags & L2:
        rng = np.random.default_rng(np.random.SeedSequence([seed, 99]))
        for x in ("q", "k"):
            scale = torch.from_numpy(rng.uniform(0.3, 4.0, inp[x].shape[:-1] + (1,)))
            t = (inp[x].double() * scale)
            t[0, 1, 0, :] = 0.0
            inp[x] = t.to(dt)
    return inp


def _oracle_view(inp, flags, dk):
    """The same inputs as the oracle sees them: the per-head gate broadcast over the key
    channels, q and k normalised in fp64 (zero rows stay zero)."""
    o = dict(inp)
    q, k, a = f64(inp["q"]), f64(inp["k"]), f64(inp["a"])
    if flags & PH:
        a = np.repeat(a[..., None], dk, axis=-1)
    norms = {}
    if flags & L2:
        for name, x in (("q", q), ("k", k)):
            n = np.linalg.norm(x, axis=-1, keepdims=True)
            norms[name] = n
            x /= np.where(n > 0, n, 1.0)
    o["q"], o["k"], o["a"] = q, k, a
    return o, norms


def _fwd_check(ops, w, seed, flags, tol):
    inp = _raw_inputs(w, seed, flags)
    d = to_device(inp)
    o, S = ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                         chunk=w.chunk, signed_gate=w.signed_gate | flags,
                         o_dtype=torch.float32)
    torch.cuda.synchronize()
    ov, _ = _oracle_view(inp, flags, w.dk)
    cu = inp.get("cu_seqlens")
    ro, rS = oracle.ckda_fwd(ov["q"], ov["k"], f64(inp["v"]), ov["a"], f64(inp["b"]),
                             f64(inp["S0"]), cu_seqlens=None if cu is None else cu.numpy(),
                             signed_gate=w.signed_gate)
    assert_close(f64(o), ro, tol, "o")
    assert_close(f64(S), rS, tol, "S_T")


@pytest.mark.parametrize("flags", [PH, L2, PH | L2], ids=["per_head", "l2norm", "both"])
@pytest.mark.parametrize("sg", [0, 1])
def test_exact_forward(cuda_lib, flags, sg):
    w = synth.CKDA_SPREAD.with_(B=2, T=150, H=2, dk=64, dv=64, chunk=32, io_dtype="f32",
                                o_dtype="f32", signed_gate=sg)
    _fwd_check(cuda_lib, w, seed=20 + sg, flags=flags, tol=TOL_FP32)


@pytest.mark.parametrize("flags", [PH, L2, PH | L2], ids=["per_head", "l2norm", "both"])
@pytest.mark.parametrize("base", [synth.KDA_STD, synth.CKDA_SPREAD], ids=["kda", "ckda"])
def test_tensor_core_forward(cuda_lib, flags, base):
    w = base.with_(B=2, T=300, H=3)
    _fwd_check(cuda_lib, w, seed=30, flags=flags, tol=TOL_BF16)


def test_tensor_core_varlen_per_head(cuda_lib):
    lens = (0, 1, 63, 64, 65, 130)
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens))
    _fwd_check(cuda_lib, w, seed=31, flags=PH | L2, tol=TOL_BF16)


@pytest.mark.parametrize("flags", [PH, PH | L2], ids=["per_head", "both"])
def test_tensor_core_per_head_fast_decay(cuda_lib, flags):
    """A per-head gate that forgets fast (the fast channel's logits, N(-2, 1)): every key
    channel decays by about 2^-211 per chunk, so all take a reference and chunks are cut."""
    w = synth.KDA_FAST.with_(B=2, T=300, H=3)
    _fwd_check(cuda_lib, w, seed=32, flags=flags, tol=TOL_BF16)


def test_tensor_core_segments_with_flags(cuda_lib):
    """Both flags on a packed batch whose longest sequence is cut into four segments (test
    hook): the segments from the identity (v = 0) normalise q and k and broadcast the gate
    like every other unit."""
    lens = (1400, 300, 0, 90)
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens))
    cuda_lib.debug_segment_split(1, 4)
    try:
        _fwd_check(cuda_lib, w, seed=33, flags=PH | L2, tol=TOL_BF16)
    finally:
        cuda_lib.debug_segment_split(0, 0)


@pytest.mark.parametrize("flags", [PH, L2, PH | L2], ids=["per_head", "l2norm", "both"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode(cuda_lib, flags, io):
    w = synth.DECODE.with_(B=3, H=4, io_dtype=io, o_dtype="f32")
    steps = 10
    dec = synth.make_decode(w, seed=40, steps=steps)
    if flags & PH:
        dec["a"] = dec["a"][..., 0].contiguous()
    if flags & L2:
        rng = np.random.default_rng(41)
        for x in ("q", "k"):
            sc = torch.from_numpy(rng.uniform(0.3, 4.0, dec[x].shape[:-1] + (1,)))
            dec[x] = (dec[x].double() * sc).to(dec[x].dtype)
    d = to_device(dec)
    S = d["S"].clone()
    outs = []
    for t in range(steps):
        outs.append(cuda_lib.decode_step(d["q"][t], d["k"][t], d["v"][t], d["a"][t], d["b"][t], S,
                                         signed_gate=1 | flags, o_dtype=torch.float32))
    torch.cuda.synchronize()
    # the oracle: one sequence of `steps` tokens per head from the initial state
    seq = lambda x: np.ascontiguousarray(f64(x).swapaxes(0, 1))
    q, k, a = seq(dec["q"]), seq(dec["k"]), seq(dec["a"])
    if flags & PH:
        a = np.repeat(a[..., None], w.dk, axis=-1)
    if flags & L2:
        for x in (q, k):
            n = np.linalg.norm(x, axis=-1, keepdims=True)
            x /= np.where(n > 0, n, 1.0)
    ro, rS = oracle.ckda_fwd(q, k, seq(dec["v"]), a, seq(dec["b"]), f64(dec["S"]), signed_gate=1)
    tol = TOL_FP32 if io == "f32" else TOL_BF16
    assert_close(f64(torch.stack(outs)), ro.swapaxes(0, 1), tol, "o")
    assert_close(f64(S), rS, tol, "S")


@pytest.mark.parametrize("flags", [PH, L2, PH | L2], ids=["per_head", "l2norm", "both"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward(cuda_lib, flags, io):
    w = synth.CKDA_SPREAD.with_(B=2, T=100, H=2, dk=64, dv=32, io_dtype=io, o_dtype="f32")
    inp = _raw_inputs(w, 50, flags)
    rng = np.random.default_rng(51)
    dO = torch.from_numpy(rng.standard_normal(inp["v"].shape)).float()
    dS_T = torch.from_numpy(rng.standard_normal((w.B, w.H, w.dk, w.dv)) * 0.1).float()
    d = to_device(inp)
    got = cuda_lib.chunk_bwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], None,
                             dO=dO.cuda(), dS_T=dS_T.cuda(), signed_gate=1 | flags)
    torch.cuda.synchronize()
    ov, norms = _oracle_view(inp, flags, w.dk)
    gq, gk, gv, ga, gb, gS0 = oracle.ckda_bwd(ov["q"], ov["k"], f64(inp["v"]), ov["a"],
                                              f64(inp["b"]), f64(inp["S0"]), dO=f64(dO),
                                              dS_T=f64(dS_T), signed_gate=1)
    if flags & L2:
        def chain(dx, x, n):
            return (dx - x * (x * dx).sum(-1, keepdims=True)) / np.where(n > 0, n, np.inf)
        gq, gk = chain(gq, ov["q"], norms["q"]), chain(gk, ov["k"], norms["k"])
    if flags & PH:
        ga = ga.sum(-1)
    for name, g, r in zip(("dq", "dk", "dv", "da", "db", "dS0"), got, (gq, gk, gv, ga, gb, gS0)):
        assert_close(f64(g), r, TOL_BWD, name)
