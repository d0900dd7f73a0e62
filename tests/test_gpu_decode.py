"""Parity of the recurrent decode step (``ckda_decode_step`` through the C ABI)
against the fp64 oracle, over many successive steps."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL_BF16, TOL_FP32, assert_close, f64, to_device
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu
INF = float("inf")


def run_steps(ops, inp, signed_gate, o_dtype=None, heads=None):
    d = to_device(inp)
    S = d["S"].clone()
    outs = []
    for t in range(d["q"].shape[0]):
        outs.append(ops.decode_step(d["q"][t], d["k"][t], d["v"][t], d["a"][t], d["b"][t], S,
                                    signed_gate=signed_gate, o_dtype=o_dtype))
    torch.cuda.synchronize()
    return torch.stack(outs), S


def oracle_steps(inp, signed_gate, heads=None):
    """Oracle over all steps; heads = optional flat (b*H + h) index list."""
    steps, B, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    sel = torch.arange(B * H) if heads is None else torch.as_tensor(np.asarray(heads))
    q, k, a = (f64(inp[x].reshape(steps, B * H, dk)[:, sel]) for x in ("q", "k", "a"))
    v = f64(inp["v"].reshape(steps, B * H, dv)[:, sel])
    b = f64(inp["b"].reshape(steps, B * H)[:, sel])
    S = f64(inp["S"].reshape(B * H, dk, dv)[sel])[None]
    os = []
    for t in range(steps):
        o, S = oracle.decode_step(q[t][None], k[t][None], v[t][None], a[t][None], b[t][None], S,
                                  signed_gate)
        os.append(o[0])
    return np.stack(os), S[0]


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16), (128, 128), (16, 128)])
def test_decode_fp32_dims(cuda_lib, dk, dv):
    w = synth.DECODE.with_(B=3, H=5, dk=dk, dv=dv, io_dtype="f32", o_dtype="f32")
    inp = synth.make_decode(w, seed=1, steps=12)
    o, S = run_steps(cuda_lib, inp, 1)
    ro, rS = oracle_steps(inp, 1)
    assert_close(f64(o).reshape(ro.shape), ro, TOL_FP32, "o")
    assert_close(f64(S).reshape(rS.shape), rS, TOL_FP32, "S")


@pytest.mark.parametrize("signed_gate", [0, 1])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16], ids=["o_f32", "o_bf16"])
def test_decode_bf16_128_steps(cuda_lib, signed_gate, o_dtype):
    w = synth.DECODE.with_(B=4, H=6, signed_gate=signed_gate,
                           gate="spread" if signed_gate else "std",
                           strength="spread" if signed_gate else "std")
    inp = synth.make_decode(w, seed=2, steps=128)
    o, S = run_steps(cuda_lib, inp, signed_gate, o_dtype=o_dtype)
    ro, rS = oracle_steps(inp, signed_gate)
    assert_close(f64(o).reshape(ro.shape), ro, TOL_BF16, "o", bf16_out=o_dtype == torch.bfloat16)
    assert_close(f64(S).reshape(rS.shape), rS, TOL_BF16, "S")


def test_decode_degenerate(cuda_lib):
    """Logits at +-inf and 0: alpha in {0, +-1}, beta in {0, 2}, exact."""
    w = synth.DECODE.with_(B=2, H=3, dk=32, dv=32, io_dtype="f32", o_dtype="f32")
    inp = synth.make_decode(w, seed=3, steps=6)
    a, b = inp["a"], inp["b"]
    a[0, :, :, :5] = INF
    a[1, :, :, :5] = -INF
    a[2, :, :, 5:9] = 0.0
    b[3] = INF
    b[4] = -INF
    o, S = run_steps(cuda_lib, inp, 1)
    ro, rS = oracle_steps(inp, 1)
    assert_close(f64(o).reshape(ro.shape), ro, TOL_FP32, "o")
    assert_close(f64(S).reshape(rS.shape), rS, TOL_FP32, "S")


def test_prefill_then_decode(cuda_lib):
    """Decode steps continuing a prefill's state equal a longer prefill."""
    w = synth.CKDA_SPREAD.with_(B=2, T=100, H=2, io_dtype="f32", o_dtype="f32")
    inp = to_device(synth.make_prefill(w, seed=4))
    o_full, S_full = cuda_lib.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"],
                                        inp["S0"], chunk=64, signed_gate=1)
    T1 = 90
    sl = lambda x: x[:, :T1].contiguous()
    _, S = cuda_lib.chunk_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["a"]),
                              sl(inp["b"]), inp["S0"], chunk=64, signed_gate=1)
    for t in range(T1, 100):
        step = lambda x: x[:, t].contiguous()
        od = cuda_lib.decode_step(step(inp["q"]), step(inp["k"]), step(inp["v"]), step(inp["a"]),
                                  step(inp["b"]), S, signed_gate=1)
        assert_close(f64(od), f64(o_full[:, t]), 1e-5, f"o step {t}")
    torch.cuda.synchronize()
    assert_close(f64(S), f64(S_full), 1e-5, "S")


def test_full_decode_whole(cuda_lib):
    """The full decode workload (B=256, H=32, d=128, 128 steps, state updated in place) in the
    benchmark's launch configuration, every head and step.  The oracle is run as one
    128-token sequence per head starting from the initial state: decode steps continuing a
    state equal the longer sequential run (pinned in the oracle's tests), and the sequential
    oracle parallelises over heads.  Blocks of 32 batch rows bound host memory."""
    w = synth.DECODE
    inp = synth.make_decode(w, seed=0)
    o, S = run_steps(cuda_lib, inp, 1, o_dtype=torch.float32)
    o, S = o.cpu(), S.cpu()
    steps = inp["q"].shape[0]
    for b0 in range(0, w.B, 32):
        sl = slice(b0, b0 + 32)
        seq = lambda x: f64(x[:, sl].transpose(0, 1))          # [32, steps, H, d]
        ro, rS = oracle.ckda_fwd(seq(inp["q"]), seq(inp["k"]), seq(inp["v"]), seq(inp["a"]),
                                 f64(inp["b"][:, sl].transpose(0, 1)), f64(inp["S"][sl]),
                                 signed_gate=1)
        assert_close(f64(o[:, sl]), ro.transpose(1, 0, 2, 3), TOL_BF16, f"o rows {b0}..")
        assert_close(f64(S[sl]), rS, TOL_BF16, f"S rows {b0}..")
    assert steps == 128


@pytest.mark.parametrize("signed_gate", [3, 4], ids=["gate_range", "strength_range"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_single_range_variants(cuda_lib, signed_gate, io):
    """The gate range or the strength range widened alone (CKDA review, Figure 6)."""
    w = synth.DECODE.with_(B=2, H=5, signed_gate=signed_gate, gate="spread", strength="spread",
                           io_dtype=io, o_dtype="f32")
    inp = synth.make_decode(w, seed=5, steps=24)
    o, S = run_steps(cuda_lib, inp, signed_gate)
    ro, rS = oracle_steps(inp, signed_gate)
    tol = TOL_FP32 if io == "f32" else TOL_BF16
    assert_close(f64(o).reshape(ro.shape), ro, tol, "o")
    assert_close(f64(S).reshape(rS.shape), rS, tol, "S")
