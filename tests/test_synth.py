"""The seeded input generator follows its stated recipe: deterministic per seed, one
independent stream per tensor, and the distributions of the CKDA review's workloads
("Method steps", step 1: standard and spread initialisation, bimodal strength)."""
import numpy as np
import pytest
import torch

from linear_rnn_ckda_b200 import synth

W = synth.KDA_STD.with_(B=2, T=512, H=4)


def f(x):
    return x.to(torch.float64).numpy()


def test_deterministic_per_seed():
    a, b = synth.make_prefill(W, seed=3), synth.make_prefill(W, seed=3)
    for k in "qkvab":
        assert torch.equal(a[k], b[k]), k
    c = synth.make_prefill(W, seed=4)
    assert not torch.equal(a["q"], c["q"])


def test_streams_are_independent():
    """Changing one tensor's distribution leaves the others' draws untouched."""
    a = synth.make_prefill(W, seed=1)
    b = synth.make_prefill(W.with_(gate="spread", strength="spread"), seed=1)
    for k in "qkv":
        assert torch.equal(a[k], b[k]), k
    assert not torch.equal(a["a"], b["a"])


def test_shapes_and_dtypes():
    d = synth.make_prefill(W, seed=0)
    assert d["q"].shape == (2, 512, 4, 128) and d["q"].dtype == torch.bfloat16
    assert d["v"].shape == (2, 512, 4, 128) and d["b"].shape == (2, 512, 4)
    assert d["b"].dtype == torch.float32
    assert d["S0"] is None and d["cu_seqlens"] is None
    d = synth.make_prefill(synth.TINY_CKDA_FP32, seed=0)
    assert d["q"].dtype == torch.float32 and d["q"].shape == (1, 64, 1, 16)


def test_unit_keys_and_queries():
    d = synth.make_prefill(W, seed=0)
    for k in "qk":
        n = np.linalg.norm(f(d[k]), axis=-1)
        assert np.abs(n - 1).max() < 1e-2, k       # unit before the bf16 rounding


@pytest.mark.parametrize("gate,moments", [("std", (4.0, 1.0)), ("tiny", (0.0, 1.5))])
def test_gate_logits_normal(gate, moments):
    a = f(synth.make_prefill(W.with_(gate=gate), seed=0)["a"]).ravel()
    mu, sd = moments
    assert abs(a.mean() - mu) < 0.01 and abs(a.std() - sd) < 0.01


def test_spread_gate_and_strength_mixtures():
    d = synth.make_prefill(W.with_(gate="spread", strength="spread"), seed=0)
    a = f(d["a"]).ravel()
    pos, neg = a[a > 0], a[a < 0]
    assert abs(pos.size / a.size - 0.5) < 0.01                  # fair coin
    assert abs(pos.mean() - 3.0) < 0.05 and abs(neg.mean() + 3.0) < 0.05
    b = f(d["b"]).ravel()
    assert abs((b > 0).mean() - 0.5) < 0.02
    assert abs(b[b > 0].mean() - 2.0) < 0.02 and abs(b[b > 0].std() - 0.5) < 0.02


def test_values_strength_and_state():
    d = synth.make_prefill(W.with_(s0=True), seed=0)
    v = f(d["v"]).ravel()
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    b = f(d["b"]).ravel()
    assert abs(b.mean()) < 0.03 and abs(b.std() - 1.0) < 0.03
    S0 = f(d["S0"])
    assert S0.shape == (2, 4, 128, 128) and abs(S0.std() - 0.02) < 5e-4


def test_varlen_lengths_and_offsets():
    lens = synth.varlen_lengths(0)
    assert len(lens) == 17 and lens[-1] == 65536
    assert all(512 <= x <= 8192 for x in lens[:16])
    w = synth.CKDA_SPREAD.with_(H=2, seq_lens=(0, 5, 70), T=75)
    d = synth.make_prefill(w, seed=0)
    assert d["cu_seqlens"].dtype == torch.int32
    assert d["cu_seqlens"].tolist() == [0, 0, 5, 75]
    assert d["q"].shape == (1, 75, 2, 128) and d["S0"].shape == (3, 2, 128, 128)


def test_decode_inputs():
    w = synth.DECODE.with_(B=4, H=3)
    d = synth.make_decode(w, seed=0, steps=5)
    assert d["q"].shape == (5, 4, 3, 128) and d["b"].shape == (5, 4, 3)
    assert d["S"].shape == (4, 3, 128, 128) and d["S"].dtype == torch.float32
    assert abs(f(d["S"]).std() - 0.02) < 1e-3


def test_fast_forgetting_recipe():
    """Every fourth key channel has logits N(-2, 1), the others N(4, 1)."""
    w = synth.KDA_FAST.with_(B=1, T=2048, H=4, io_dtype="f32")
    a = synth.make_prefill(w, seed=3)["a"].double()
    fast, slow = a[..., 0::4], a[..., 1::4]
    assert abs(fast.mean().item() + 2.0) < 0.02 and abs(fast.std().item() - 1.0) < 0.02
    assert abs(slow.mean().item() - 4.0) < 0.02 and abs(slow.std().item() - 1.0) < 0.02
