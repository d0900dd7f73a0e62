"""ckda_chunk_fwd_noalloc: the forward for callers that cannot allocate device
memory (a runtime with a fixed memory plan, or C code with no device
allocator).  It must give the same results as ckda_chunk_fwd with a
caller-allocated workspace, call after call, although every call reuses the
library's one fixed scratch array.  Collected last so that a run stopping at
the first failure has already run every other test."""
import ctypes

import pytest
import torch

from helpers import TOL_BF16, TOL_FP32, assert_close, f64, to_device
from linear_rnn_ckda_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(ops, d, w, o, S_T):
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    B, T, H, dk = d["q"].shape
    cu = d["cu_seqlens"]
    n_seqs = 0 if cu is None else cu.numel() - 1
    rc = ops.load().ckda_chunk_fwd_noalloc(
        P(d["q"]), P(d["k"]), P(d["v"]), P(d["a"]), P(d["b"]), P(d["S0"]), P(cu), n_seqs, B, T, H,
        dk, d["v"].shape[-1], w.chunk, w.signed_gate, 1 if d["q"].dtype == torch.bfloat16 else 0,
        1 if o.dtype == torch.bfloat16 else 0, P(o), P(S_T),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, ops.status_string(rc)


@pytest.mark.parametrize("w,tol", [
    (synth.CKDA_SPREAD.with_(B=2, T=300, H=3, o_dtype="f32"), TOL_BF16),          # tensor-core path
    (synth.TINY_CKDA_FP32.with_(B=2, T=77, H=2, s0=True), TOL_FP32),             # fp32 path
    (synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=(5, 64, 0, 130), T=199, o_dtype="f32"), TOL_BF16),
], ids=["bf16_d128", "fp32_d16", "varlen"])
def test_noalloc_matches_workspace_entry_point(cuda_lib, w, tol):
    for call, seed in enumerate((40, 41)):          # two calls in a row, different inputs
        d = to_device(synth.make_prefill(w, seed))
        ref_o, ref_S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"],
                                          d["cu_seqlens"], chunk=w.chunk, signed_gate=w.signed_gate,
                                          o_dtype=torch.float32 if w.o_dtype == "f32" else None)
        o = torch.full_like(ref_o, float("nan"))
        S_T = torch.full_like(ref_S, float("nan"))
        _noalloc(cuda_lib, d, w, o, S_T)
        torch.cuda.synchronize()
        assert cuda_lib.noalloc_status() == 0, call
        assert_close(f64(o), f64(ref_o), tol, f"o call {call}")
        assert_close(f64(S_T), f64(ref_S), tol, f"S_T call {call}")


def test_noalloc_status_reports_bad_offsets_then_clears(cuda_lib):
    """Offsets that do not end at T make the kernel skip the bad sequence and record
    CKDA_ERR_SEQLENS in the scratch's status word, readable with ckda_noalloc_status; the
    next good call starts from a cleared status and matches ckda_chunk_fwd."""
    w = synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=(50, 70), T=120, o_dtype="f32")
    d = to_device(synth.make_prefill(w, seed=42))
    bad = dict(d, cu_seqlens=torch.tensor([0, 50, 110], dtype=torch.int32, device="cuda"))
    o = torch.zeros(1, 120, 2, 128, device="cuda")
    S_T = torch.zeros(2, 2, 128, 128, device="cuda")
    _noalloc(cuda_lib, bad, w, o, S_T)
    assert cuda_lib.noalloc_status() == -6          # CKDA_ERR_SEQLENS
    ref_o, ref_S = cuda_lib.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"],
                                      d["cu_seqlens"], signed_gate=1, o_dtype=torch.float32)
    o = torch.full_like(ref_o, float("nan"))
    S_T = torch.full_like(ref_S, float("nan"))
    _noalloc(cuda_lib, d, w, o, S_T)
    assert cuda_lib.noalloc_status() == 0
    assert_close(f64(o), f64(ref_o), TOL_BF16, "o after a failed call")
    assert_close(f64(S_T), f64(ref_S), TOL_BF16, "S_T after a failed call")


def test_noalloc_rejects_bad_arguments(cuda_lib):
    """Validation is the workspace entry point's: a bad chunk size is refused."""
    w = synth.TINY_CKDA_FP32.with_(chunk=8)
    d = to_device(synth.make_prefill(synth.TINY_CKDA_FP32, 0))
    o = torch.empty_like(d["v"])
    S_T = torch.empty(1, 1, 16, 16, device="cuda")
    with pytest.raises(AssertionError, match="chunk"):
        _noalloc(cuda_lib, d, w, o, S_T)
