"""Parity of the chunkwise backward (``ckda_chunk_bwd`` through the C ABI) against the fp64
oracle's backward (the plain reverse of the token step, pinned by finite differences and
closed forms) on the same seeded inputs: the gradients of sum dO . o + sum dS_T . S_T with
respect to q, k, v, the gate and strength logits and S0.

The backward computes in fp32 throughout (exact gate products, exact zero gates), so on the
same input values it meets an fp32-level bar whatever the input dtype: TOL_BWD, the forward's
fp32 bar widened tenfold for the longer chains of products a gradient goes through (the
inverse of I + A, the gate gradient's sums over row pairs)."""
import numpy as np
import pytest
import torch

from helpers import TOL_BF16, assert_close, compare_bwd_whole, f64, to_device, GRAD_NAMES
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu
INF = float("inf")
TOL_BWD = 1e-4


def _cotangents(inp, n_seqs, seed, do_dtype=torch.float32):
    """Seeded dO ~ N(0, 1) and dS_T ~ N(0, 0.1) shaped like o and S_T."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 77]))
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    dO = torch.from_numpy(rng.standard_normal((B, T, H, dv))).to(do_dtype)
    dS_T = torch.from_numpy(rng.standard_normal((n_seqs, H, dk, dv)) * 0.1).float()
    return dO, dS_T


def run_bwd(ops, inp, dO, dS_T, signed_gate, want_dS0=True):
    d = to_device(inp)
    g = ops.chunk_bwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                      dO=None if dO is None else dO.cuda(),
                      dS_T=None if dS_T is None else dS_T.cuda(), signed_gate=signed_gate,
                      want_dS0=want_dS0)
    torch.cuda.synchronize()
    return g


def check(ops, w, seed, tol=TOL_BWD, do_dtype=torch.float32, inp=None):
    inp = synth.make_prefill(w, seed) if inp is None else inp
    dO, dS_T = _cotangents(inp, w.n_seqs, seed, do_dtype)
    got = run_bwd(ops, inp, dO, dS_T, w.signed_gate)
    return compare_bwd_whole(got, inp, dO, dS_T, w.signed_gate, tol)


@pytest.mark.parametrize("signed_gate", [0, 1, 2, 3, 4])
def test_tiny_all_gate_forms(cuda_lib, signed_gate):
    w = synth.TINY_CKDA_FP32.with_(B=2, T=70, H=2, s0=True, signed_gate=signed_gate,
                                   gate="spread" if signed_gate != 2 else "tiny")
    inp = synth.make_prefill(w, seed=signed_gate)
    if signed_gate == 2:   # raw gates in [-1, 1], strengths in [0, 2]
        inp["a"] = torch.tanh(inp["a"])
        inp["b"] = 2 * torch.sigmoid(inp["b"])
    check(cuda_lib, w, seed=signed_gate, inp=inp)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16)])
def test_dims_fp32(cuda_lib, dk, dv):
    w = synth.CKDA_SPREAD.with_(B=2, T=100, H=2, dk=dk, dv=dv, io_dtype="f32", o_dtype="f32")
    check(cuda_lib, w, seed=dk + dv)


@pytest.mark.parametrize("base", [synth.KDA_STD, synth.CKDA_SPREAD], ids=["kda_std", "ckda_spread"])
@pytest.mark.parametrize("do_dtype", [torch.float32, torch.bfloat16], ids=["dO_f32", "dO_bf16"])
def test_bf16_inputs(cuda_lib, base, do_dtype):
    check(cuda_lib, base.with_(B=2, T=200, H=2), seed=3, do_dtype=do_dtype)


def test_varlen_edges(cuda_lib):
    lens = (0, 1, 31, 32, 33, 100, 0, 65)
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens), io_dtype="f32",
                                o_dtype="f32")
    check(cuda_lib, w, seed=4)


def test_optional_arguments(cuda_lib):
    """dO absent (only dS_T drives the gradients), dS_T absent, and no dS0 requested."""
    w = synth.CKDA_SPREAD.with_(B=2, T=90, H=2, io_dtype="f32", o_dtype="f32")
    inp = synth.make_prefill(w, seed=5)
    dO, dS_T = _cotangents(inp, w.n_seqs, 5)
    for use_dO, use_dS in ((False, True), (True, False)):
        a, b = (dO if use_dO else None), (dS_T if use_dS else None)
        got = run_bwd(cuda_lib, inp, a, b, 1)
        compare_bwd_whole(got, inp, a, b, 1, TOL_BWD)
    got = run_bwd(cuda_lib, inp, dO, dS_T, 1, want_dS0=False)
    assert got[5] is None
    compare_bwd_whole(got, inp, dO, dS_T, 1, TOL_BWD)


def _raw_case(T, dk, dv, alpha, beta, seed=0, H=1):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, H, dk))
    k = rng.standard_normal((1, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, dv))
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.1
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).float()
    return {"q": t(q), "k": t(k), "v": t(v), "a": t(alpha), "b": t(beta), "S0": t(S0),
            "cu_seqlens": None}


def test_degenerate_gates(cuda_lib):
    """Exact zero gates (one channel, a whole row), gates of +-1, strong decay (products far
    below fp32's range) and strengths of 0 and 2, raw gates; then the same through logits
    of +-inf and 0 in the KDA and CKDA forms.  An exact zero gate's gradient is the
    derivative at that gate."""
    rng = np.random.default_rng(5)
    T, dk, dv = 110, 32, 32
    alpha = rng.uniform(-1, 1, (1, T, 1, dk))
    alpha[0, 10, 0, :] = 0.0
    alpha[0, 20:30, 0, 3] = 0.0
    alpha[0, 40:60, 0, 5] = -1.0
    alpha[0, 70:90, 0, :8] = 1e-4
    alpha[0, 100:, 0, 9] = 1.0
    beta = rng.uniform(0, 2, (1, T, 1))
    beta[0, 5] = 0.0
    beta[0, 6:9] = 2.0
    inp = _raw_case(T, dk, dv, alpha, beta)
    w = synth.TINY_CKDA_FP32.with_(B=1, T=T, H=1, dk=dk, dv=dv, signed_gate=2)
    check(cuda_lib, w, seed=6, inp=inp)
    for sg in (0, 1):
        a = rng.standard_normal((1, T, 1, dk)) * 3
        a[0, 3, 0, :4] = INF
        a[0, 4, 0, :4] = -INF
        a[0, 7, 0, 4:8] = 0.0
        b = rng.standard_normal((1, T, 1))
        b[0, 11], b[0, 12] = INF, -INF
        inp = _raw_case(T, dk, dv, a, b, seed=7)
        check(cuda_lib, w.with_(signed_gate=sg), seed=8, inp=inp)


def test_full_kda_std_whole(cuda_lib):
    """The KDA workload B=4, T=4096, H=16, d=128 (bf16 inputs), every gradient element."""
    check(cuda_lib, synth.KDA_STD, seed=0, do_dtype=torch.bfloat16)


@pytest.mark.slow
def test_full_ckda_spread_whole(cuda_lib):
    """The CKDA spread-init workload B=8, T=8192, H=16, d=128 with S0, every gradient element."""
    check(cuda_lib, synth.CKDA_SPREAD, seed=0, do_dtype=torch.bfloat16)
