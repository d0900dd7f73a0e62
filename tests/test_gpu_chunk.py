"""Parity of the chunkwise forward (``ckda_chunk_fwd`` through the C ABI)
against the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

from helpers import (TOL_BF16, TOL_FP32, assert_close, compare_prefill_whole, f64, oracle_prefill,
                     to_device)
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu
INF = float("inf")


def run_gpu(ops, inp, w, chunk=None, o_dtype=None, S0_alias=False):
    d = to_device(inp)
    S_T = None
    if S0_alias and d["S0"] is not None:
        S_T = d["S0"]
    o, S = ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                         chunk=chunk or w.chunk, signed_gate=w.signed_gate,
                         o_dtype=o_dtype, S_T=S_T)
    torch.cuda.synchronize()
    return o, S


def check(ops, w, seed=0, tol=None, chunk=None, o_dtype=None):
    inp = synth.make_prefill(w, seed)
    o, S = run_gpu(ops, inp, w, chunk, o_dtype)
    ro, rS = oracle_prefill(inp, w.signed_gate)
    tol = tol or (TOL_FP32 if w.io_dtype == "f32" and o.dtype == torch.float32 else TOL_BF16)
    eo, _ = assert_close(f64(o), ro, tol, w.name + " o", bf16_out=o.dtype == torch.bfloat16)
    es, _ = assert_close(f64(S), rS, tol, w.name + " S_T")
    return eo, es


def close(x, ref, tol, what=""):
    """assert_close on a GPU tensor (fp32 or bf16) against an fp64 oracle array."""
    return assert_close(f64(x), ref, tol, what, bf16_out=x.dtype == torch.bfloat16)


def test_tiny_ckda_fp32(cuda_lib):
    """The tiny CKDA workload: B=1, H=1, T=64, d=16, fp32, chunk 16, seed 0."""
    check(cuda_lib, synth.TINY_CKDA_FP32)


@pytest.mark.parametrize("dk,dv", [(16, 16), (16, 64), (32, 32), (64, 16), (64, 128), (128, 32),
                                   (128, 128)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_dims_and_chunks_fp32(cuda_lib, dk, dv, chunk):
    w = synth.TINY_CKDA_FP32.with_(name="dims", B=2, T=77, H=3, dk=dk, dv=dv, chunk=chunk, s0=True,
                                   gate="spread", strength="spread")
    check(cuda_lib, w, seed=1)


@pytest.mark.parametrize("base", [synth.KDA_STD, synth.CKDA_SPREAD], ids=["kda_std", "ckda_spread"])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16], ids=["o_f32", "o_bf16"])
def test_bf16_small(cuda_lib, base, o_dtype):
    """Same distributions as the full workloads on a smaller grid (several chunks, ragged tail)."""
    w = base.with_(B=2, T=300, H=3)
    check(cuda_lib, w, seed=2, o_dtype=o_dtype)


def test_fp32_io_d128(cuda_lib):
    w = synth.CKDA_SPREAD.with_(B=1, T=200, H=2, io_dtype="f32", o_dtype="f32")
    check(cuda_lib, w, seed=3, tol=TOL_FP32)


@pytest.mark.parametrize("dk,dv,chunk", [(64, 64, 32), (128, 128, 16), (128, 128, 32),
                                         (128, 64, 64), (32, 128, 64), (16, 16, 16)])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16], ids=["o_f32", "o_bf16"])
def test_exact_path_bf16_inputs(cuda_lib, dk, dv, chunk, o_dtype):
    """bf16 q/k/v/a on the exact CUDA-core kernel (every shape the tensor-core kernel does not
    take: head sizes other than 128, or chunks of 16 and 32).  Its arithmetic is fp32
    throughout, so with an fp32 output it meets the fp32 bar against the oracle on the same
    bf16 values; a bf16 output meets the bf16 bar."""
    w = synth.CKDA_SPREAD.with_(name=f"exact_bf16_{dk}x{dv}_c{chunk}", B=2, T=150, H=2, dk=dk,
                                dv=dv, chunk=chunk)
    check(cuda_lib, w, seed=14, o_dtype=o_dtype,
          tol=TOL_FP32 if o_dtype == torch.float32 else TOL_BF16)
    check(cuda_lib, w.with_(signed_gate=0, gate="std", strength="std", s0=False), seed=15,
          o_dtype=o_dtype, tol=TOL_FP32 if o_dtype == torch.float32 else TOL_BF16)


def test_varlen_edge_lengths(cuda_lib):
    """Packed batch with empty, length-1, ragged and chunk-multiple sequences."""
    lens = (0, 1, 63, 64, 65, 200, 0, 129)
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens), io_dtype="f32",
                                o_dtype="f32")
    inp = synth.make_prefill(w, seed=4)
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, w.signed_gate)
    close(o, ro, TOL_FP32, "o")
    close(S, rS, TOL_FP32, "S_T")
    S0 = f64(inp["S0"])
    assert np.array_equal(f64(S)[0], S0[0]) and np.array_equal(f64(S)[6], S0[6])


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


@pytest.mark.parametrize("chunk", [16, 64])
def test_degenerate_gates(cuda_lib, chunk):
    """Exact zeros, +-1, strong decay and beta at 0 and 2 (raw gates), and the
    same through +-inf logits in both gate forms."""
    rng = np.random.default_rng(5)
    T, dk, dv = 150, 32, 32
    alpha = rng.uniform(-1, 1, (1, T, 1, dk))
    alpha[0, 10, 0, :] = 0.0            # a full state wipe
    alpha[0, 20:30, 0, 3] = 0.0         # one channel held at zero
    alpha[0, 40:60, 0, 5] = -1.0
    alpha[0, 70:90, 0, :8] = 1e-4       # strong decay (products underflow fp32)
    alpha[0, 100:, 0, 9] = 1.0
    beta = rng.uniform(0, 2, (1, T, 1))
    beta[0, 5] = 0.0
    beta[0, 6:9] = 2.0
    inp = _raw_case(T, dk, dv, alpha, beta)
    w = synth.TINY_CKDA_FP32.with_(B=1, T=T, H=1, dk=dk, dv=dv, chunk=chunk, signed_gate=2)
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, 2)
    close(o, ro, TOL_FP32, "o raw")
    close(S, rS, TOL_FP32, "S_T raw")
    # logits at +-inf and 0 in the CKDA and KDA forms
    for sg in (0, 1):
        a = rng.standard_normal((1, T, 1, dk)) * 3
        a[0, 3, 0, :4] = INF
        a[0, 4, 0, :4] = -INF
        a[0, 7, 0, 4:8] = 0.0
        b = rng.standard_normal((1, T, 1))
        b[0, 11], b[0, 12] = INF, -INF
        inp = _raw_case(T, dk, dv, a, b, seed=6)
        o, S = run_gpu(cuda_lib, inp, w.with_(signed_gate=sg))
        ro, rS = oracle_prefill(inp, sg)
        close(o, ro, TOL_FP32, f"o sg{sg}")
        close(S, rS, TOL_FP32, f"S_T sg{sg}")


def test_exact_rotation_on_gpu(cuda_lib):
    """alpha = (-1, 1), beta = 2 (logits -inf/+inf/+inf), k = (cos t, sin t) in a 16-dim
    head (other channels alpha = 1, k = 0): the top-left 2x2 block of the state
    is rotated by 2 * sum(t) and the rest is unchanged."""
    T, dk, dv, m = 48, 16, 16, 5
    rng = np.random.default_rng(7)
    x = rng.integers(0, m, size=T)
    th = np.pi * x / m
    k = np.zeros((1, T, 1, dk))
    k[0, :, 0, 0], k[0, :, 0, 1] = np.cos(th), np.sin(th)
    a = np.full((1, T, 1, dk), INF)
    a[0, :, 0, 0] = -INF
    inp = {"q": torch.zeros(1, T, 1, dk), "k": torch.from_numpy(k).float(),
           "v": torch.zeros(1, T, 1, dv), "a": torch.from_numpy(a).float(),
           "b": torch.full((1, T, 1), INF), "S0": torch.eye(dk).reshape(1, 1, dk, dv).contiguous(),
           "cu_seqlens": None}
    w = synth.TINY_CKDA_FP32.with_(B=1, T=T, H=1, dk=dk, dv=dv, chunk=16, signed_gate=1)
    _, S = run_gpu(cuda_lib, inp, w)
    S = f64(S)[0, 0]
    ang = 2 * np.pi * (x.sum() % m) / m
    R = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
    assert np.allclose(S[:2, :2], R, atol=1e-5)
    assert np.allclose(S[2:, 2:], np.eye(dk - 2), atol=1e-6)


def test_state_alias_and_resume(cuda_lib):
    """S_T may alias S0; run(T1) then run(T2) from its state equals run(T1 + T2)."""
    w = synth.CKDA_SPREAD.with_(B=2, T=190, H=2, io_dtype="f32", o_dtype="f32")
    inp = synth.make_prefill(w, seed=8)
    o_full, S_full = run_gpu(cuda_lib, inp, w)
    T1 = 77
    first = {k: (v[:, :T1].contiguous() if k in "qkvab" else v) for k, v in inp.items()}
    second = {k: (v[:, T1:].contiguous() if k in "qkvab" else v) for k, v in inp.items()}
    d1 = to_device(first)
    o1, S1 = cuda_lib.chunk_fwd(d1["q"], d1["k"], d1["v"], d1["a"], d1["b"], d1["S0"], chunk=64,
                                signed_gate=1)
    d2 = to_device(second)
    o2, S2 = cuda_lib.chunk_fwd(d2["q"], d2["k"], d2["v"], d2["a"], d2["b"], S1, chunk=64,
                                signed_gate=1, S_T=S1)           # in place
    torch.cuda.synchronize()
    assert S2.data_ptr() == S1.data_ptr()
    assert_close(f64(torch.cat([o1, o2], 1)), f64(o_full), 1e-5, "o resumed")
    assert_close(f64(S2), f64(S_full), 1e-5, "S_T resumed")


def test_chunk_size_invariance(cuda_lib):
    w = synth.CKDA_SPREAD.with_(B=1, T=257, H=2, io_dtype="f32", o_dtype="f32")
    inp = synth.make_prefill(w, seed=9)
    outs = [run_gpu(cuda_lib, inp, w, chunk=c) for c in (16, 32, 64)]
    for o, S in outs[1:]:
        assert_close(f64(o), f64(outs[0][0]), 1e-5, "o across chunk sizes")
        assert_close(f64(S), f64(outs[0][1]), 1e-5, "S_T across chunk sizes")


@pytest.mark.parametrize("io", ["f32", "bf16"], ids=["exact", "tensor_core"])
def test_bad_seqlens_sets_status(cuda_lib, io):
    """Decreasing offsets: the kernel (the exact one) or the unit planner (tensor-core path)
    skips the bad sequences and records the error."""
    w = synth.CKDA_SPREAD.with_(B=1, H=1, seq_lens=(10, 10), T=20, io_dtype=io, o_dtype="f32")
    inp = to_device(synth.make_prefill(w, seed=10))
    cu = torch.tensor([0, 15, 12], dtype=torch.int32, device="cuda")  # ends below start
    ws = cuda_lib.new_workspace(1, 20, 1, 128, 128, 64, 2)
    cuda_lib.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"], cu,
                       signed_gate=1, workspace=ws)
    assert cuda_lib.workspace_status(ws) == -6
    cuda_lib.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["S0"],
                       inp["cu_seqlens"], signed_gate=1, workspace=ws)
    assert cuda_lib.workspace_status(ws) == 0


# ---------------------------------------------------------------- full-size workloads
# The full workloads, whole tensors (every sequence, head and token), in the launch
# configuration the benchmark times (bf16 io, bf16 o, chunk 64), against the oracle on the
# same inputs.


def _whole(ops, w, seed=0):
    inp = synth.make_prefill(w, seed)
    o, S = run_gpu(ops, inp, w)
    return compare_prefill_whole(o, S, inp, w.signed_gate, TOL_BF16,
                                 bf16_out=o.dtype == torch.bfloat16)


def test_full_kda_std_whole(cuda_lib):
    """KDA workload B=4, T=4096, H=16, d=128."""
    _whole(cuda_lib, synth.KDA_STD)


@pytest.mark.slow
def test_full_ckda_spread_whole(cuda_lib):
    """CKDA spread-init workload B=8, T=8192, H=16, d=128, S0 ~ N(0, 0.02)."""
    _whole(cuda_lib, synth.CKDA_SPREAD)


@pytest.mark.slow
def test_full_varlen_whole(cuda_lib):
    """Varlen CKDA workload: H=32, 16 lengths U{512..8192} + 65,536 packed with cu_seqlens."""
    _whole(cuda_lib, synth.varlen_workload(0))


# ---------------------------------------------------------------- tensor-core path
# bf16 q/k/v/a with dk = dv = 128 and chunk 64 run on the tcgen05 kernel.


def _bf16_raw_case(T, alpha_logit, b_logit, seed, H=2, S0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, H, 128))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((1, T, H, 128))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, 128))
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x)).float().to(torch.bfloat16)
    return {"q": bf(q), "k": bf(k), "v": bf(v), "a": bf(alpha_logit),
            "b": torch.from_numpy(np.ascontiguousarray(b_logit)).float(),
            "S0": torch.from_numpy(rng.standard_normal((1, H, 128, 128)) * 0.02).float()
            if S0 else None, "cu_seqlens": None}


@pytest.mark.parametrize("sg", [0, 1])
def test_tc_degenerate_gates(cuda_lib, sg):
    """Zero gates, +-1 gates, beta at 0 and 2 and strong decay on the bf16 d=128 path:
    chunks whose gate products leave [2^-100, 2^100] take the exact token path."""
    T, H = 333, 2
    rng = np.random.default_rng(20 + sg)
    a = rng.standard_normal((1, T, H, 128)) * 2 + (0 if sg else 3)
    a[0, 5, 0, :] = -INF if sg == 0 else 0.0        # alpha = 0: full wipe in head 0
    a[0, 70:75, 1, 10:20] = -INF if sg == 0 else 0.0
    a[0, 140:150, 0, :] = INF                      # alpha = 1
    if sg:
        a[0, 150:160, 1, :] = -INF                 # alpha = -1
    a[0, 200:264, 0, :32] = 1e-3 if sg else -60.0  # strong decay: products underflow
    b = rng.standard_normal((1, T, H))
    b[0, 7, :], b[0, 8, :] = INF, -INF
    inp = _bf16_raw_case(T, a, b, seed=30 + sg)
    w = synth.CKDA_SPREAD.with_(B=1, T=T, H=H, signed_gate=sg, o_dtype="f32")
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, sg)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_varlen_edges(cuda_lib):
    lens = (0, 1, 63, 64, 65, 130, 0, 7)
    w = synth.CKDA_SPREAD.with_(B=1, H=3, seq_lens=lens, T=sum(lens), o_dtype="f32")
    inp = synth.make_prefill(w, seed=11)
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, 1)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")
    S0 = f64(inp["S0"])
    assert np.array_equal(f64(S)[0], S0[0]) and np.array_equal(f64(S)[6], S0[6])


def test_tc_matches_simt(cuda_lib):
    """The tcgen05 path (bf16 inputs) and the exact fp32 path (the same values as
    fp32) agree within the bf16 tolerance."""
    w = synth.KDA_STD.with_(B=2, T=257, H=2, o_dtype="f32")
    inp = synth.make_prefill(w, seed=12)
    o_tc, S_tc = run_gpu(cuda_lib, inp, w)
    inp32 = {k: (v.float() if v is not None and v.dtype == torch.bfloat16 else v)
             for k, v in inp.items()}
    o_ex, S_ex = run_gpu(cuda_lib, inp32, w.with_(io_dtype="f32"))
    assert_close(f64(o_tc), f64(o_ex), TOL_BF16, "o tc vs exact")
    assert_close(f64(S_tc), f64(S_ex), TOL_BF16, "S_T tc vs exact")


def test_tc_state_alias_and_chunk_boundaries(cuda_lib):
    """S_T aliasing S0 in place; T = 64, 128 and 129 exercise one, two and a ragged chunk."""
    for T in (64, 128, 129):
        w = synth.CKDA_SPREAD.with_(B=2, T=T, H=2, o_dtype="f32")
        inp = synth.make_prefill(w, seed=13 + T)
        ro, rS = oracle_prefill(inp, 1)
        o, S = run_gpu(cuda_lib, inp, w, S0_alias=True)
        close(o, ro, TOL_BF16, f"o T={T}")
        close(S, rS, TOL_BF16, f"S_T T={T}")


@pytest.mark.parametrize("sg", [0, 1])
def test_tc_small_gate_logits(cuda_lib, sg):
    """Gate logits near zero on the bf16 d=128 path (CKDA gates of either sign and size
    below 0.05, KDA gates near 1/2), mixed into large ones so that the chunks stay on the
    factorised path: the gates' products must still match the oracle."""
    T, H = 300, 2
    rng = np.random.default_rng(40 + sg)
    a = rng.standard_normal((1, T, H, 128)) + np.where(rng.random((1, T, H, 128)) < 0.5, 3.0, -3.0)
    small = rng.random((1, T, H, 128)) < 0.1
    a[small] = rng.uniform(-0.1, 0.1, size=int(small.sum()))
    b = rng.standard_normal((1, T, H))
    inp = _bf16_raw_case(T, a, b, seed=50 + sg)
    w = synth.CKDA_SPREAD.with_(B=1, T=T, H=H, signed_gate=sg, o_dtype="f32")
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, sg)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_fast_forgetting_channels(cuda_lib):
    """KDA gates with every fourth key channel forgetting fast (logits N(-2, 1)): those
    channels decay by about 2^-211 over a chunk, so they take a power-of-two reference and some
    chunks are cut short; the result matches the oracle whatever each chunk did."""
    w = synth.KDA_FAST.with_(B=2, T=400, H=2, o_dtype="f32")
    check(cuda_lib, w, seed=16)


@pytest.mark.parametrize("sg", [0, 1])
def test_tc_range_cuts(cuda_lib, sg):
    """Decay that leaves the factorisation's range at known row groups: gates of 2^-8 per row
    in one channel (a chunk fits 24 rows), of 2^-20 (8 rows), of 2^-30 (not even 8 rows: token
    by token), zero gates 0, 7, 8 and 63 rows apart, and stretches of ordinary gates between
    them, so that chunks start at unaligned rows and the sequence ends inside a cut chunk.
    Every row of o and S_T matches the oracle."""
    T, H = 701, 2
    rng = np.random.default_rng(60 + sg)
    a = rng.standard_normal((1, T, H, 128)) * 0.5 + (3.0 if sg == 0 else 4.0)
    if sg:
        a *= np.where(rng.random(a.shape) < 0.5, 1.0, -1.0)

    def logit(log2_alpha):  # a whose gate is 2^log2_alpha (KDA: sigma(a); CKDA: tanh(a/2))
        x = 2.0 ** log2_alpha
        return math.log(x / (1 - x)) if sg == 0 else 2 * math.atanh(x)

    a[0, 0:300, 0, 3] = logit(-8)
    a[0, 300:400, :, 7] = logit(-20)
    a[0, 520:545, 1, 11] = logit(-30)
    zero = -INF if sg == 0 else 0.0
    for r in (448, 455, 456, 511):
        a[0, r, r % 2, 9 + r % 5] = zero
    a[0, 640:701, 0, 20] = logit(-8)      # a cut chunk runs into the end of the sequence
    b = rng.standard_normal((1, T, H))
    inp = _bf16_raw_case(T, a, b, seed=70 + sg)
    w = synth.CKDA_SPREAD.with_(B=1, T=T, H=H, signed_gate=sg, o_dtype="f32")
    o, S = run_gpu(cuda_lib, inp, w)
    ro, rS = oracle_prefill(inp, sg)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_handoff_positions(cuda_lib):
    """Units handed to the kernel with references at their first chunk (head 0), in the middle
    (head 1, fast gates from row 150) and in the ragged last chunk (head 2, from row 262 of
    273); S_T written over S0.  The workspace header's hand-off count says all three moved."""
    T, H = 273, 3
    rng = np.random.default_rng(80)
    a = rng.standard_normal((1, T, H, 128)) * 0.5 + 3.0
    fast = math.log(2.0 ** -5 / (1 - 2.0 ** -5))      # KDA gate 2^-5: 320 bits per 64 rows
    a[0, :, 0, 17] = fast
    a[0, 150:, 1, 40:44] = fast
    a[0, 262:, 2, 99] = -60.0                          # 2^-87 per row: not even 8 rows fit
    b = rng.standard_normal((1, T, H))
    inp = _bf16_raw_case(T, a, b, seed=81, H=H)
    w = synth.KDA_STD.with_(B=1, T=T, H=H, o_dtype="f32")
    d = to_device(inp)
    ws = cuda_lib.new_workspace(1, T, H, 128, 128, 64, 0, torch.device("cuda"))
    S = d["S0"].clone()
    o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], S, None, chunk=64,
                              signed_gate=0, o_dtype=torch.float32, S_T=S, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[64:68].view(torch.int32).item()) == 3
    ro, rS = oracle_prefill(inp, 0)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_fast_forgetting_without_handoff(cuda_lib):
    """With only the 256-byte workspace header there is no room for the hand-off to the kernel
    with references: chunks past the plain kernel's range run token by token, exactly."""
    w = synth.KDA_FAST.with_(B=2, T=200, H=2, o_dtype="f32")
    inp = synth.make_prefill(w, seed=18)
    d = to_device(inp)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], None, chunk=64,
                              signed_gate=w.signed_gate, o_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    ro, rS = oracle_prefill(inp, w.signed_gate)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_fast_forgetting_varlen_alias(cuda_lib):
    """The fast-forgetting gates in a packed batch (cut chunks cross no sequence boundary)
    with S_T written over S0."""
    lens = (0, 1, 63, 64, 65, 200, 7, 333)
    w = synth.KDA_FAST.with_(B=1, H=2, seq_lens=lens, T=sum(lens), o_dtype="f32")
    inp = synth.make_prefill(w, seed=17)
    ro, rS = oracle_prefill(inp, w.signed_gate)
    o, S = run_gpu(cuda_lib, inp, w, S0_alias=True)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


# ---------------------------------------------------------------- segments of long sequences
# The longest sequences of a batch may be cut into segments: the first launch runs each segment
# from a zero state and from the identity with v = 0 (its affine state map), a small kernel
# chains the maps, and the second launch runs the segments from their true starting states.


def _seg_header(ws):
    """The plan's header in the workspace (byte 128): unit counts of the two launches, the
    number of cut sequences and each one's segment count."""
    h = ws[128:176].view(torch.int32).cpu().numpy()
    return {"n1": int(h[0]), "n3": int(h[1]), "nsplit": int(h[2]),
            "m": [int(h[4 + 4 * i]) for i in range(2)]}


def _run_cut(ops, w, inp, n_split, nseg, S0_alias=True):
    d = to_device(inp)
    N = len(w.seq_lens) if w.seq_lens is not None else w.B
    ws = ops.new_workspace(w.B, w.T, w.H, 128, 128, 64,
                           N if w.seq_lens is not None else 0, torch.device("cuda"))
    S = d["S0"].clone() if S0_alias else None
    ops.debug_segment_split(n_split, nseg)
    try:
        o, S = ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                             chunk=64, signed_gate=w.signed_gate, o_dtype=torch.float32, S_T=S,
                             workspace=ws)
        torch.cuda.synchronize()
    finally:
        ops.debug_segment_split(0, 0)
    assert ops.workspace_status(ws) == 0
    return o, S, _seg_header(ws)


@pytest.mark.parametrize("n_split,nseg", [(1, 3), (2, 4), (2, 8)])
@pytest.mark.parametrize("sg", [0, 1])
def test_tc_segments_forced(cuda_lib, n_split, nseg, sg):
    """A packed batch whose one or two longest sequences are cut (test hook) into 3, 4 or 8
    segments, the last one ragged, with empty and one-token sequences beside them and S_T
    written over S0: every row of o and S_T matches the oracle, and the plan's header says
    how many sequences were cut and into how many segments."""
    lens = (1500, 0, 2333, 64, 700, 1)
    base = synth.CKDA_SPREAD if sg else synth.KDA_STD
    w = base.with_(B=1, H=3, seq_lens=lens, T=sum(lens), o_dtype="f32", s0=True)
    inp = synth.make_prefill(w, seed=90 + nseg + sg)
    o, S, hdr = _run_cut(cuda_lib, w, inp, n_split, nseg)
    assert hdr["nsplit"] == n_split
    for i, ln in enumerate(sorted(lens, reverse=True)[:n_split]):
        ch = -(-ln // 64)
        seg = -(-ch // nseg)
        assert hdr["m"][i] == -(-ch // seg)
    ro, rS = oracle_prefill(inp, sg)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


def test_tc_segments_without_states(cuda_lib):
    """A cut packed batch with no S0 (segment 0 starts from zero) and no S_T requested (the
    last segment writes no end state): o matches the oracle row for row."""
    lens = (2000, 333, 64)
    w = synth.KDA_STD.with_(B=1, H=2, seq_lens=lens, T=sum(lens), o_dtype="bf16", s0=False)
    inp = synth.make_prefill(w, seed=97)
    d = to_device(inp)
    ws = cuda_lib.new_workspace(1, w.T, w.H, 128, 128, 64, len(lens), torch.device("cuda"))
    cuda_lib.debug_segment_split(1, 5)
    try:
        o, S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], None, d["cu_seqlens"],
                                  chunk=64, signed_gate=0, workspace=ws, want_state=False)
        torch.cuda.synchronize()
    finally:
        cuda_lib.debug_segment_split(0, 0)
    assert S is None and cuda_lib.workspace_status(ws) == 0
    assert _seg_header(ws)["nsplit"] == 1 and _seg_header(ws)["m"][0] == 5
    ro, _ = oracle_prefill(inp, 0)
    close(o, ro, TOL_BF16, "o")


def test_tc_segments_fast_forgetting(cuda_lib):
    """Cut sequences whose gates forget fast: units of both launches (segments from zero, from
    the identity, from the chained states) are handed to the kernel with references."""
    lens = (900, 1300, 50)
    w = synth.KDA_FAST.with_(B=1, H=2, seq_lens=lens, T=sum(lens), o_dtype="f32", s0=True)
    inp = synth.make_prefill(w, seed=95)
    o, S, hdr = _run_cut(cuda_lib, w, inp, 2, 5)
    assert hdr["nsplit"] == 2
    ro, rS = oracle_prefill(inp, w.signed_gate)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")


@pytest.mark.parametrize("B,T,H", [(1, 16384, 4), (2, 8192, 2)])
def test_tc_segments_chosen_by_cost(cuda_lib, B, T, H):
    """Few long sequences and few heads (4 walks of 256 chunks, or 4 of 128, on 148 SMs): the
    cost model cuts every sequence by itself (unpacked rows, so each unit addresses its own
    batch row); without a workspace large enough for the plan the same call runs uncut.  Both
    match the oracle."""
    w = synth.KDA_STD.with_(B=B, T=T, H=H, o_dtype="f32", s0=True)
    inp = synth.make_prefill(w, seed=96 + B)
    o, S, hdr = _run_cut(cuda_lib, w, inp, 0, 0, S0_alias=False)
    assert hdr["nsplit"] == B and min(hdr["m"][:B]) >= 3
    ro, rS = oracle_prefill(inp, w.signed_gate)
    close(o, ro, TOL_BF16, "o")
    close(S, rS, TOL_BF16, "S_T")
    d = to_device(inp)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")   # the header alone: no plan
    o2, S2 = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], None, chunk=64,
                                signed_gate=w.signed_gate, o_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert _seg_header(ws)["nsplit"] == 0 and _seg_header(ws)["n1"] == 0
    close(o2, ro, TOL_BF16, "o uncut")
    close(S2, rS, TOL_BF16, "S_T uncut")


@pytest.mark.parametrize("signed_gate", [3, 4], ids=["gate_range", "strength_range"])
def test_single_range_variants(cuda_lib, signed_gate):
    """The gate range or the strength range widened alone (CKDA review, Figure 6) on both
    prefill paths: exact fp32 (d=64, chunk 32) and tensor-core bf16 (d=128, chunk 64)."""
    w32 = synth.CKDA_SPREAD.with_(B=2, T=150, H=2, dk=64, dv=64, chunk=32,
                                  signed_gate=signed_gate, io_dtype="f32", o_dtype="f32")
    check(cuda_lib, w32, seed=7, tol=TOL_FP32)
    wtc = synth.CKDA_SPREAD.with_(B=2, T=300, H=3, signed_gate=signed_gate, o_dtype="f32")
    check(cuda_lib, wtc, seed=8)


# ---------------------------------------------------------------- bounded waits
# Every wait of the tensor-core kernel is bounded; when one runs out the unit gives up,
# lets its copies and products finish, frees its tensor memory and records
# CKDA_ERR_TIMEOUT.  The test hook adds a wait that runs out (on a barrier nothing arrives
# on) at the start of one chunk of every unit that reaches it.


@pytest.mark.parametrize("chunk_index", [0, 1, 3])
def test_tc_wait_timeout_recovers(cuda_lib, chunk_index):
    lens = (40, 300, 130)        # 1, 5 and 3 chunks
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=lens, T=sum(lens), o_dtype="f32")
    inp = synth.make_prefill(w, seed=60)
    # an exact zero gate (CKDA logit 0) in head 0 at local token 67 of sequence 1: that
    # unit's chunk 1 runs token by token, so the hook meets the slow path too
    inp["a"][0, lens[0] + 67, 0, :] = 0.0
    d = to_device(inp)
    ro, rS = oracle_prefill(inp, 1)
    ws = cuda_lib.new_workspace(1, w.T, w.H, 128, 128, 64, len(lens))
    o = torch.full((1, w.T, w.H, 128), float("nan"), device="cuda")
    S = torch.full((len(lens), w.H, 128, 128), float("nan"), device="cuda")
    try:
        cuda_lib.debug_wait_injection(chunk_index, 200_000)     # 0.2 ms bound
        cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                           signed_gate=1, o_dtype=torch.float32, o=o, S_T=S, workspace=ws)
        assert cuda_lib.workspace_status(ws) == -8      # CKDA_ERR_TIMEOUT
    finally:
        cuda_lib.debug_wait_injection(-1, 0)
    # sequences that end before that chunk never met the wait: complete and correct
    cu = [0] + list(np.cumsum(lens))
    for n, L in enumerate(lens):
        if (L + 63) // 64 <= chunk_index:
            close(o[:, cu[n]:cu[n + 1]], ro[:, cu[n]:cu[n + 1]], TOL_BF16, f"o seq {n}")
            close(S[n], rS[n], TOL_BF16, f"S_T seq {n}")
    # the context is intact: a normal call on the same stream and workspace is correct
    o2, S2 = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                                signed_gate=1, o_dtype=torch.float32, workspace=ws)
    assert cuda_lib.workspace_status(ws) == 0
    close(o2, ro, TOL_BF16, "o after recovery")
    close(S2, rS, TOL_BF16, "S_T after recovery")
