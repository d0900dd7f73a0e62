"""DeltaProduct2 (two rank-one delta-rule updates per token, the gate once; CKDA review,
"Research motivation" and "Experimental results" (5)) on the exact forward kernel and on
decode, against the oracle's plain DeltaProduct form on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL_BF16, TOL_FP32, assert_close, f64, to_device
from linear_rnn_ckda_b200 import ops as ops_mod
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu
P2 = ops_mod.DELTA_PRODUCT2


def _inputs(w, seed):
    """The workload's q, a, S0 and a second key, value and strength per token: k, v, b drawn
    from the workload recipe for 2T tokens and laid out as [B, T, 2, H, .]."""
    base = synth.make_prefill(w, seed)
    twice = synth.make_prefill(w.with_(T=2 * w.T, seq_lens=None, B=w.B), seed + 1000)
    B, T, H = w.B, w.T, w.H
    out = dict(base)
    out["k"] = twice["k"].reshape(B, T, 2, H, w.dk).contiguous()
    out["v"] = twice["v"].reshape(B, T, 2, H, w.dv).contiguous()
    out["b"] = twice["b"].reshape(B, T, 2, H).contiguous()
    return out


@pytest.mark.parametrize("dk,dv,chunk", [(16, 16, 16), (64, 32, 32), (128, 128, 64)])
@pytest.mark.parametrize("sg", [0, 1, 3])
def test_product2_forward_fp32(cuda_lib, dk, dv, chunk, sg):
    w = synth.CKDA_SPREAD.with_(B=2, T=75, H=2, dk=dk, dv=dv, chunk=chunk, io_dtype="f32",
                                o_dtype="f32", signed_gate=sg)
    inp = _inputs(w, seed=60 + sg)
    d = to_device(inp)
    o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], None, chunk=chunk,
                              signed_gate=sg | P2)
    torch.cuda.synchronize()
    ro, rS = oracle.ckda_fwd_product(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["a"]),
                                     f64(inp["b"]), f64(inp["S0"]), signed_gate=sg)
    assert_close(f64(o), ro, TOL_FP32, "o")
    assert_close(f64(S), rS, TOL_FP32, "S_T")


def test_product2_forward_bf16_flags(cuda_lib):
    """bf16 inputs, d = 128, chunk 64 (the shapes the tensor-core kernel takes for one update
    per token run here on the exact kernel), with the per-head gate and in-kernel q/k
    normalisation."""
    w = synth.CKDA_SPREAD.with_(B=2, T=100, H=2)
    inp = _inputs(w, seed=70)
    inp["a"] = inp["a"][..., 0].contiguous()
    d = to_device(inp)
    flags = 1 | P2 | ops_mod.GATE_PER_HEAD | ops_mod.QK_L2NORM
    o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], None, chunk=64,
                              signed_gate=flags, o_dtype=torch.float32)
    torch.cuda.synchronize()
    q, k = f64(inp["q"]), f64(inp["k"])
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a = np.repeat(f64(inp["a"])[..., None], w.dk, axis=-1)
    ro, rS = oracle.ckda_fwd_product(q, k, f64(inp["v"]), a, f64(inp["b"]), f64(inp["S0"]),
                                     signed_gate=1)
    assert_close(f64(o), ro, TOL_BF16, "o")
    assert_close(f64(S), rS, TOL_BF16, "S_T")


def test_product2_varlen(cuda_lib):
    lens = (0, 1, 7, 8, 9, 40, 0, 33)
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens), dk=32, dv=32, chunk=16,
                                io_dtype="f32", o_dtype="f32")
    base = synth.make_prefill(w, 80)
    T = sum(lens)
    twice = synth.make_prefill(w.with_(seq_lens=None, T=2 * T), 81)
    inp = dict(base)
    inp["k"] = twice["k"].reshape(1, T, 2, 2, 32).contiguous()
    inp["v"] = twice["v"].reshape(1, T, 2, 2, 32).contiguous()
    inp["b"] = twice["b"].reshape(1, T, 2, 2).contiguous()
    d = to_device(inp)
    o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                              chunk=16, signed_gate=1 | P2)
    torch.cuda.synchronize()
    ro, rS = oracle.ckda_fwd_product(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["a"]),
                                     f64(inp["b"]), f64(inp["S0"]),
                                     cu_seqlens=inp["cu_seqlens"].numpy(), signed_gate=1)
    assert_close(f64(o), ro, TOL_FP32, "o")
    assert_close(f64(S), rS, TOL_FP32, "S_T")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_product2_decode_matches_prefill_oracle(cuda_lib, io):
    """Decode steps with two updates each, continuing a state, against the oracle's
    DeltaProduct form over the same tokens."""
    w = synth.DECODE.with_(B=3, H=4, io_dtype=io, o_dtype="f32")
    steps = 8
    dec = synth.make_decode(w, seed=90, steps=steps)
    extra = synth.make_decode(w.with_(B=2 * w.B), seed=91, steps=steps)
    k = extra["k"].reshape(steps, w.B, 2, w.H, w.dk).contiguous()
    v = extra["v"].reshape(steps, w.B, 2, w.H, w.dv).contiguous()
    b = extra["b"].reshape(steps, w.B, 2, w.H).contiguous()
    d = {x: dec[x].cuda() for x in ("q", "a")}
    kd, vd, bd = k.cuda(), v.cuda(), b.cuda()
    S = dec["S"].cuda()
    outs = [cuda_lib.decode_step(d["q"][t], kd[t], vd[t], d["a"][t], bd[t], S,
                                 signed_gate=1 | P2, o_dtype=torch.float32) for t in range(steps)]
    torch.cuda.synchronize()
    sw = lambda x: np.ascontiguousarray(f64(x).swapaxes(0, 1))
    ro, rS = oracle.ckda_fwd_product(sw(dec["q"]), sw(k), sw(v), sw(dec["a"]), sw(b),
                                     f64(dec["S"]), signed_gate=1)
    tol = TOL_FP32 if io == "f32" else TOL_BF16
    assert_close(f64(torch.stack(outs)), ro.swapaxes(0, 1), tol, "o")
    assert_close(f64(S), rS, tol, "S")


def test_product2_backward_refused(cuda_lib):
    w = synth.CKDA_SPREAD.with_(B=1, T=10, H=1, dk=16, dv=16, io_dtype="f32")
    inp = to_device(_inputs(w, 95))
    with pytest.raises(ops_mod.CkdaError, match="dtype"):
        cuda_lib.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], None,
                           signed_gate=1 | P2)
