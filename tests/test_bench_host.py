"""Host-side parts of the benchmark that need no GPU: the algorithmic work per launch that
the roofline fractions divide by, and the parsing of the clock log sampled during the timed
region (the throttle reasons decide whether a number stands)."""
import os
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_rnn_ckda_b200 import synth  # noqa: E402


def test_prefill_flops_per_token_head():
    # 6 d^2 (state products) + C (3 dk + 2 dv) (intra-chunk products) + C^2 / 3 (solve), counted
    # by hand for d = 128, C = 64: 98,304 + 40,960 + 1,365.33
    assert bench.prefill_flops_per_token_head(128, 128, 64) == pytest.approx(140629.33, abs=0.01)
    assert bench.prefill_flops_per_token_head(16, 16, 16) == pytest.approx(1536 + 1280 + 85.33,
                                                                             abs=0.01)


def test_prefill_bytes_of_the_workloads():
    # KDA std, B4 T4096 H16: 262,144 token-heads x (q, k, v, a bf16 = 1,024 B + b 4 B + o bf16
    # 256 B = 1,284 B) + S_T of 64 heads (64 KB each), no S0 read
    assert bench.prefill_bytes(synth.KDA_STD) == 262144 * 1284 + 64 * 65536
    # CKDA spread, B8 T8192 H16 with S0: 1,048,576 token-heads x 1,284 B + S0 and S_T of 128 heads
    assert bench.prefill_bytes(synth.CKDA_SPREAD) == 1048576 * 1284 + 128 * 65536 * 2
    # fp32 o adds 256 B per token-head
    w = synth.KDA_STD.with_(o_dtype="f32")
    assert bench.prefill_bytes(w) == 262144 * 1540 + 64 * 65536


def test_decode_bytes_per_step():
    # B256 H32: per head the fp32 state read and written (2 x 64 KB) + q, k, v, a bf16 (1,024 B)
    # + b (4 B) + o fp32 (512 B)
    assert bench.decode_bytes(synth.DECODE) == 8192 * (131072 + 1024 + 4 + 512)


def _summary(lines):
    s = bench.ClockSampler(0)
    fd, s.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.proc = object()          # a sampler that ran (its process is not needed to parse)
    out = s.summary()
    assert not os.path.exists(s.path)
    return out


def test_clock_log_parsing():
    na, act = "Not Active", "Active"
    lines = [
        f"0, 1965, 1965, 612.10, 0x0000000000000000, {na}, {na}, {na}, {na}",
        f"0, 1830, 1965, 998.50, 0x0000000000000004, {na}, {na}, {na}, {act}",
        f"0, 1890, 1965, 990.00, 0x0000000000000004, {na}, {na}, {na}, {act}",
        "garbage line",
        f"0, [N/A], 1965, 0, 0x0, {na}, {na}, {na}, {na}",
    ]
    out = _summary(lines)
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1890
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    hot = _summary([f"0, 1400, 1965, 700, 0x8, {na}, {act}, {na}, {na}"])
    assert hot["reasons"] == ["hw_thermal_slowdown"]


def test_clock_log_absent():
    s = bench.ClockSampler(0)
    assert s.summary() is None         # nvidia-smi never started
