"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function ``include/ckda.h`` declares, and rejects bad arguments with the
documented codes before touching a device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckda.h")

from linear_rnn_ckda_b200 import build as lib_build  # noqa: E402
from linear_rnn_ckda_b200 import ops  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    lib_build.build_library()
    return ops.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ckda_\w+)\s*\(", text)))


def declared_codes():
    text = open(HEADER).read()
    return {m[0]: int(m[1]) for m in re.findall(r"#define (CKDA_\w+) \(?(-?\d+)\)?", text)}


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("ckda_chunk_fwd", "ckda_chunk_fwd_workspace_size", "ckda_decode_step",
              "ckda_status_string", "ckda_workspace_status", "ckda_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in ckda.h but not exported"
        assert name in ops.SIGNATURES, f"{name} has no binding signature"


def test_binding_codes_match_header():
    codes = declared_codes()
    assert codes["CKDA_F32"] == ops.CKDA_F32 and codes["CKDA_BF16"] == ops.CKDA_BF16


def test_status_strings(lib):
    codes = declared_codes()
    for name, code in codes.items():
        if name.startswith("CKDA_ERR") or name == "CKDA_OK":
            s = lib.ckda_status_string(code).decode()
            assert s and s != "unknown status", name
    assert lib.ckda_status_string(12345).decode() == "unknown status"
    assert lib.ckda_version() >= 100


def test_workspace_size(lib):
    """The 256-byte header; for the tensor-core shapes also the hand-off's queue (16 bytes per
    (sequence, head), rounded up to 256) and one fp32 128 x 128 state per (sequence, head)."""
    assert lib.ckda_chunk_fwd_workspace_size(1, 0, 1, 16, 16, 16, 0) == 256
    assert lib.ckda_chunk_fwd_workspace_size(2, 100, 3, 64, 64, 64, 0) == 256
    assert lib.ckda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 32, 0) == 256
    units = 4 * 16
    assert lib.ckda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 64, 0) == \
        256 + 1024 + units * 65536
    # a packed batch may have its two longest sequences cut into up to 8 segments: the unit
    # lists hold n_seqs + 2 * 13 entries (32 bytes each, two lists), the hand-off covers that
    # many units of one launch, and 2 * 13 state slots per head hold the segments' states
    entries = 3 + 26
    units = entries * 2
    assert lib.ckda_chunk_fwd_workspace_size(1, 1000, 2, 128, 128, 64, 3) == \
        256 + 1024 + units * 65536 + 2048 + 26 * 2 * 65536
    # unpacked: the plan's room only where the cost model (148 SMs) cuts; one sequence of
    # 65,536 tokens over 16 heads (16 walks of 1,024 chunks) is cut
    entries = 1 + 26
    units = entries * 16
    assert lib.ckda_chunk_fwd_workspace_size(1, 65536, 16, 128, 128, 64, 0) == \
        256 + 6912 + units * 65536 + 1792 + 26 * 16 * 65536
    no_plan = lambda B, T, H: 256 + (((B * H * 16) + 255) // 256) * 256 + B * H * 65536
    for B, T, H in ((4, 4096, 16), (8, 8192, 16), (2, 65536, 64), (1, 2048, 1)):
        assert lib.ckda_chunk_fwd_workspace_size(B, T, H, 128, 128, 64, 0) == no_plan(B, T, H)


# Fake, aligned, never-dereferenced host addresses: every call below has exactly
# one invalid argument, so validation rejects it before any CUDA call.
P = ctypes.c_void_p(1 << 20)
MIS = ctypes.c_void_p((1 << 20) + 4)     # 4-byte aligned, not 16
ODD = ctypes.c_void_p((1 << 20) + 2)     # 2-byte aligned only


def _fwd(lib, **kw):
    args = dict(q=P, k=P, v=P, a=P, b=P, S0=None, cu=None, n_seqs=0, B=1, T=8, H=1, dk=16, dv=16,
                chunk=16, sg=1, io=0, od=0, o=P, S_T=P, ws=P, wsb=256, stream=None)
    args.update(kw)
    return lib.ckda_chunk_fwd(*args.values())


def _dec(lib, **kw):
    args = dict(q=P, k=P, v=P, a=P, b=P, S=P, B=1, H=1, dk=16, dv=16, sg=1, io=0, od=0, o=P,
                stream=None)
    args.update(kw)
    return lib.ckda_decode_step(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(b=None), -1),
    (dict(dk=24), -2), (dict(dv=256), -2), (dict(H=0), -2), (dict(T=-1), -2), (dict(B=-1), -2),
    (dict(cu=P, B=2, n_seqs=1), -2),
    (dict(chunk=128), -3), (dict(chunk=8), -3),
    (dict(sg=5), -4), (dict(io=2), -4), (dict(od=-1), -4),
    (dict(k=MIS), -5), (dict(o=MIS), -5), (dict(S0=MIS), -5), (dict(S_T=MIS), -5),
    (dict(b=ODD), -5), (dict(cu=ODD), -5),
    (dict(ws=None), -7), (dict(wsb=16), -7), (dict(ws=ctypes.c_void_p((1 << 20) + 16)), -7),
    # token rows are 32-bit coordinates: B * T above 2^31 - 1 is refused
    (dict(B=2, T=1 << 30), -2), (dict(B=1 << 16, T=1 << 15), -2),
])
def test_chunk_fwd_rejects(lib, kw, code):
    assert _fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(S=None), -1), (dict(q=None), -1), (dict(dk=48), -2), (dict(H=0), -2),
    (dict(sg=-1), -4), (dict(io=5), -4), (dict(v=ODD), -5), (dict(q=ODD), -5), (dict(S=MIS), -5),
    (dict(b=ODD), -5), (dict(io=1, od=0, o=ODD), -5),
])
def test_decode_rejects(lib, kw, code):
    assert _dec(lib, **kw) == code


def test_workspace_status_rejects_null(lib):
    st = ctypes.c_int(0)
    assert lib.ckda_workspace_status(None, ctypes.byref(st), None) == -1
    assert lib.ckda_noalloc_status(None, None) == -1


def test_largest_token_count_passes_validation(lib):
    """B * T = 2^31 - 1 is inside the limit: with a too-small workspace the call gets past the
    size checks and stops at the workspace check (no CUDA call is made)."""
    assert _fwd(lib, B=1, T=(1 << 31) - 1, wsb=0) == -7


def test_noalloc_rejects_before_any_cuda_call(lib):
    """The no-allocation entry point validates like ckda_chunk_fwd (a bad chunk size)."""
    rc = lib.ckda_chunk_fwd_noalloc(P, P, P, P, P, None, None, 0, 1, 8, 1, 16, 16, 8, 1, 0, 0, P, P,
                                    None)
    assert rc == -3


def test_wait_injection_hook_is_settable(lib):
    """The test hook takes any value and is switched off again (no device work)."""
    ops.debug_wait_injection(3, 1000)
    ops.debug_wait_injection(-1, 0)


def test_binding_has_no_cpu_fallback(lib):
    x = torch.zeros(1, 8, 1, 16)
    with pytest.raises(ValueError):
        ops.chunk_fwd(x, x, x, x, torch.zeros(1, 8, 1), chunk=16)
    with pytest.raises(ValueError):
        ops.decode_step(x[:, 0], x[:, 0], x[:, 0], x[:, 0], torch.zeros(1, 1),
                        torch.zeros(1, 1, 16, 16))


# ---------------------------------------------------------------- binding argument checks
# The C ABI receives bare pointers, so the binding checks what it cannot: that every tensor
# has the shape and dtype its pointer is read or written as.

from linear_rnn_ckda_b200 import synth  # noqa: E402


@pytest.mark.parametrize("w", [synth.TINY_CKDA_FP32, synth.KDA_STD.with_(B=2, T=70, H=3),
                               synth.CKDA_SPREAD.with_(B=2, T=70, H=3, o_dtype="f32"),
                               synth.CKDA_SPREAD.with_(B=1, H=2, seq_lens=(0, 1, 65), T=66)],
                         ids=["tiny", "kda", "ckda_s0", "varlen"])
def test_binding_accepts_the_workloads(w):
    d = synth.make_prefill(w, seed=0)
    od = torch.float32 if w.o_dtype == "f32" else torch.bfloat16
    N, dv = ops.check_prefill_args(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"],
                                   d["cu_seqlens"], o_dtype=od)
    assert (N, dv) == (w.n_seqs, w.dv)
    B, T, H = d["q"].shape[:3]
    o = torch.empty(B, T, H, dv, dtype=od)
    S_T = torch.empty(N, H, w.dk, dv)
    ops.check_prefill_args(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                           o=o, S_T=S_T, o_dtype=od)
    dec = synth.make_decode(synth.DECODE.with_(B=2, H=3), seed=0, steps=2)
    assert ops.check_decode_args(dec["q"][0], dec["k"][0], dec["v"][0], dec["a"][0],
                                 dec["b"][0], dec["S"], o_dtype=torch.float32) == 128


def _prefill_bad(**over):
    w = synth.KDA_STD.with_(B=2, T=70, H=3, s0=True)
    d = synth.make_prefill(w, seed=0)
    args = dict(q=d["q"], k=d["k"], v=d["v"], a=d["a"], b=d["b"], S0=d["S0"], cu_seqlens=None)
    args.update(over)
    return args


@pytest.mark.parametrize("name,over", [
    ("k_shorter", lambda d: dict(k=d["k"][:, :60])),
    ("a_other_dtype", lambda d: dict(a=d["a"].float())),
    ("v_other_dtype", lambda d: dict(v=d["v"].float())),
    ("v_other_heads", lambda d: dict(v=d["v"][:, :, :2])),
    ("b_bf16", lambda d: dict(b=d["b"].to(torch.bfloat16))),
    ("b_per_channel", lambda d: dict(b=d["a"].float())),
    ("q_3d", lambda d: dict(q=d["q"][0])),
    ("S0_wrong_heads", lambda d: dict(S0=d["S0"][:, :2])),
    ("S0_bf16", lambda d: dict(S0=d["S0"].to(torch.bfloat16))),
    ("seqlens_int64", lambda d: dict(cu_seqlens=torch.tensor([0, 70]))),
    ("seqlens_with_batch", lambda d: dict(cu_seqlens=torch.tensor([0, 70], dtype=torch.int32))),
    ("o_wrong_dtype", lambda d: dict(o=torch.empty(2, 70, 3, 128))),
    ("o_short", lambda d: dict(o=torch.empty(2, 69, 3, 128, dtype=torch.bfloat16))),
    ("S_T_wrong", lambda d: dict(S_T=torch.empty(2, 3, 128, 64))),
])
def test_binding_rejects_mismatched_buffers(name, over):
    base = _prefill_bad()
    args = _prefill_bad(**over(base))
    with pytest.raises(ValueError):
        ops.check_prefill_args(**args)


@pytest.mark.parametrize("name,over", [
    ("k_shorter", lambda d: dict(k=d["k"][:1])),
    ("b_bf16", lambda d: dict(b=d["b"].to(torch.bfloat16))),
    ("S_wrong_dv", lambda d: dict(S=d["S"][..., :64])),
    ("S_bf16", lambda d: dict(S=d["S"].to(torch.bfloat16))),
    ("v_other_dtype", lambda d: dict(v=d["v"].float())),
    ("o_wrong_shape", lambda d: dict(o=torch.empty(2, 3, 64))),
])
def test_decode_binding_rejects_mismatched_buffers(name, over):
    dec = synth.make_decode(synth.DECODE.with_(B=2, H=3), seed=0, steps=1)
    d = {k: (v[0] if k != "S" else v) for k, v in dec.items()}
    args = dict(q=d["q"], k=d["k"], v=d["v"], a=d["a"], b=d["b"], S=d["S"])
    args.update(over(d))
    with pytest.raises(ValueError):
        ops.check_decode_args(**args)


def _bwd(lib, **kw):
    args = dict(q=P, k=P, v=P, a=P, b=P, S0=None, cu=None, n_seqs=0, B=1, T=8, H=1, dk=16, dv=16,
                sg=1, io=0, dO=P, do_dt=0, dS_T=None, dq=P, dk_=P, dv_=P, da=P, db=P, dS0=None,
                ws=P, wsb=1 << 30, stream=None)
    args.update(kw)
    return lib.ckda_chunk_bwd(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(dq=None), -1), (dict(db=None), -1), (dict(da=None), -1),
    (dict(dk=24), -2), (dict(H=0), -2), (dict(B=2, T=1 << 30), -2),
    (dict(sg=7), -4), (dict(do_dt=3), -4), (dict(io=2), -4),
    (dict(dq=MIS), -5), (dict(dO=MIS), -5), (dict(dS_T=MIS), -5), (dict(db=ODD), -5),
    (dict(ws=None), -7), (dict(wsb=256), -7),
])
def test_chunk_bwd_rejects(lib, kw, code):
    assert _bwd(lib, **kw) == code


def test_bwd_workspace_size(lib):
    """Per 32-row chunk slot and head: the state and its gradient (fp32 [dk][dv] each) and the
    chunk's record (Kr, Kd, Qr [32][dk], Li, P, M [32][32], beta [32], g [dk], fp32, rounded
    to 16 bytes), plus the 256-byte header; a packed batch allows one extra slot per
    sequence."""
    rec = 3 * 32 * 128 + 3 * 32 * 32 + 32 + 128
    per = (2 * 128 * 128 + rec) * 4 * 16
    assert lib.ckda_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 0) == 256 + 512 * per
    assert lib.ckda_chunk_bwd_workspace_size(1, 4096, 16, 128, 128, 3) == 256 + (128 + 4) * per
    rec16 = (3 * 32 * 16 + 3 * 32 * 32 + 32 + 16 + 3) // 4 * 4
    assert lib.ckda_chunk_bwd_workspace_size(1, 32, 1, 16, 48, 0) == 256 + (2 * 16 * 48 + rec16) * 4


def test_segment_cost_model(lib):
    """The segment cut's cost model, which the device planner evaluates for packed batches
    (ckda_debug_segment_choice runs it on the host).  The long-context varlen batch (16
    sequences of 512..8192 tokens and one of 65,536, 32 heads) cuts the long one into three
    segments (32 heads x 3 first-launch units fit one wave of 148 SMs; four segments would not);
    one 65,536-token sequence over 16 heads is cut into six; two of 8,192 over 2 heads both
    into eight.  Equal-length batches that already fill the GPU, batches whose total work
    outweighs their longest walk, and sequences under 48 chunks are not cut."""
    from linear_rnn_ckda_b200 import synth

    assert ops.debug_segment_choice(synth.varlen_lengths(0), 32) == (1, [3])
    assert ops.debug_segment_choice([65536], 16) == (1, [6])
    assert ops.debug_segment_choice([8192, 8192], 2) == (2, [8, 8])
    assert ops.debug_segment_choice([4096] * 4, 16) == (0, [])
    assert ops.debug_segment_choice([8192] * 8, 16) == (0, [])
    assert ops.debug_segment_choice([65536] + [8192] * 200, 32) == (0, [])
    assert ops.debug_segment_choice([3008, 64, 64], 1) == (0, [])   # 47 chunks
    assert ops.debug_segment_choice([3009, 64, 64], 1) == (1, [8])   # 48 chunks
    assert ops.debug_segment_choice([], 4) == (0, [])
    # half the SMs: six segments would need two waves in both launches (walk 4 x 171 chunks);
    # five take two waves in the first launch only (3 x 205)
    assert ops.debug_segment_choice([65536], 16, sm_count=74) == (1, [5])
    with pytest.raises(ops.CkdaError):
        ops.debug_segment_choice([100, -1], 4)
    with pytest.raises(ops.CkdaError):
        ops.debug_segment_choice([64] * 1025, 4)
