#!/usr/bin/env python3
"""Benchmark of the KDA / Complex-KDA hot path on B200.

Prints ONE JSON line (rank 0).  The headline is the chunkwise prefill
(``ckda_chunk_fwd``) on the largest single-GPU workload, the long-context
varlen CKDA batch: H=32, dk=dv=128, 16 packed sequences of lengths uniform in
[512, 8192] plus one of 65,536 tokens (cu_seqlens), per-sequence S0 ~ N(0, 0.02),
chunk 64, bf16 q/k/v/a, bf16 o, fp32 state.  ``value`` is prefill tokens/s for
the whole job; one step = one ``ckda_chunk_fwd`` call over the whole packed
batch with its inputs resident in HBM.  The same run reports, each with its own
roofline: the KDA workload (B=4, T=4096, H=16), the CKDA spread-init workload
(B=8, T=8192, H=16, S0), the CKDA/KDA throughput ratio of the same kernel, and
the decode step (``ckda_decode_step``, B=256, H=32, fp32 state in place) as
state GB/s against HBM.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workloads on
its own seeded data (independent (sequence, head) units, no data-path
collective); ``value`` = all ranks' tokens / max-over-ranks time ("weak").

``--impl reference`` times the fp64 CPU oracle (the only other arm; there is
no installable reference implementation) on a bounded sample of the headline
workload, on the host cores of rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from linear_rnn_ckda_b200 import synth  # noqa: E402

# the metric as the headline's definition states it (both arms print it verbatim)
METRIC = "chunk-fwd prefill tokens/s + % tensor roofline; decode state GB/s vs HBM peak"
HEADLINE = synth.varlen_workload(0)
KDA = synth.KDA_STD
SPREAD = synth.CKDA_SPREAD
DECODE = synth.DECODE

# Algorithmic counts per unit (d = dk = dv = 128, chunk C = 64):
#   prefill FLOP per token-head = 6 d^2 + C (3 dk + 2 dv) + C^2 / 3
#   prefill bytes per token-head = q + k + v + a (bf16) + b (fp32) + o (bf16)
#   plus S_T (fp32 d^2) per (sequence, head), and S0 when the workload has one
#   decode bytes per head-step = read + write of the fp32 state + q, k, v, a, b, o


def prefill_flops_per_token_head(dk, dv, C):
    return 6 * dk * dv + C * (3 * dk + 2 * dv) + C * C / 3.0


def prefill_bytes(w):
    io = 2 if w.io_dtype == "bf16" else 4
    ob = 2 if w.o_dtype == "bf16" else 4
    per_th = io * (3 * w.dk + w.dv) + 4 + ob * w.dv
    th = w.tokens * w.H
    state = w.n_seqs * w.H * w.dk * w.dv * 4 * (2 if w.s0 else 1)
    return th * per_th + state


def decode_bytes(w):
    io = 2 if w.io_dtype == "bf16" else 4
    ob = 2 if w.o_dtype == "bf16" else 4
    heads = w.B * w.H
    return heads * (2 * w.dk * w.dv * 4 + io * (3 * w.dk + w.dv) + 4 + ob * w.dv)


PROFILED = os.path.join(ROOT, "profiles", "roofline_traffic.json")
CSRC = os.path.join(ROOT, "linear_rnn_ckda_b200", "csrc")


def source_hash(files):
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(key):
    """DRAM bytes per launch of one kernel on one workload (``key`` = "kernel/workload") from
    the committed ncu capture, or None when there is none or the kernel's sources changed
    after the capture."""
    try:
        with open(PROFILED) as f:
            rec = json.load(f)[key]
        if source_hash(rec["sources"]) != rec["source_sha256"]:
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock and throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9], parts[4]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, x in enumerate(r[2]) if x == "Active"})
        sm = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_loop(fn, steps, warmup, world, stream):
    """Device time of `steps` calls of fn (after `warmup`), CUDA events on `stream`."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return ev0.elapsed_time(ev1)  # ms


def _oracle_run(inp, signed_gate, threads):
    """The oracle on one host input dict (upcast to fp64); returns its wall time."""
    import numpy as np

    import oracle

    f = lambda t: None if t is None else np.ascontiguousarray(t.to(torch.float64).numpy())
    cu = inp.get("cu_seqlens")
    args = [f(inp[x]) for x in "qkvab"]
    oracle.build()
    t0 = time.perf_counter()
    oracle.ckda_fwd(*args, f(inp.get("S0")), cu_seqlens=None if cu is None else cu.numpy(),
                    signed_gate=signed_gate, threads=threads, want_o=True)
    return time.perf_counter() - t0


def _slice_sequences(inp, lo, hi):
    """Sequences lo..hi-1 of a packed (cu_seqlens) input dict, repacked."""
    cu = inp["cu_seqlens"]
    t0, t1 = int(cu[lo]), int(cu[hi])
    out = {x: inp[x][:, t0:t1].contiguous() for x in "qkvab"}
    out["S0"] = None if inp.get("S0") is None else inp["S0"][lo:hi].contiguous()
    out["cu_seqlens"] = (cu[lo:hi + 1] - cu[lo]).to(torch.int32)
    return out


def cpu_baseline_sample(host, w, seqs):
    """The oracle, as it stands, on sequences ``seqs`` (a range) of the packed workload ``w``
    (all heads) with every host core: (tokens/s, cores, description)."""
    cores = os.cpu_count() or 1
    sub = _slice_sequences(host, seqs.start, seqs.stop)
    tokens = int(sub["cu_seqlens"][-1])
    dt = _oracle_run(sub, w.signed_gate, cores)
    units = (seqs.stop - seqs.start) * w.H
    desc = (f"sequences {seqs.start}..{seqs.stop - 1} of {w.name} ({tokens} tokens x {w.H} heads, "
            f"{units} (sequence, head) units), fp64 sequential per unit, {dt:.2f} s wall")
    return tokens / dt, min(cores, units), desc


def run_reference(args, world, rank):
    """The reference arm: the oracle on the host cores, on a bounded sample of the headline
    workload per step (two of its sequences, regenerated from the same recipe), with the
    headline's metric, unit and config."""
    if rank != 0:
        return
    w = HEADLINE
    lens = w.seq_lens
    cores = os.cpu_count() or 1
    times, toks = [], []
    for i in range(args.warmup + args.steps):
        j = (2 * i) % 16
        sw = w.with_(seq_lens=(lens[j], lens[j + 1]), T=lens[j] + lens[j + 1])
        inp = synth.make_prefill(sw, seed=1000 + i)
        dt = _oracle_run(inp, w.signed_gate, cores)
        if i >= args.warmup:
            times.append(dt)
            toks.append(sw.tokens)
    tot = sum(times)
    value = sum(toks) / tot
    sample = (f"per step two of the 16 short sequences of {w.name} (lengths from its length "
              f"list, regenerated from the same recipe; {w.H} heads each), fp64 sequential per "
              f"(sequence, head) unit")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * tot / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(cores, 2 * w.H),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def headline_config(w):
    return {"workload": w.name, "H": w.H, "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
            "signed_gate": w.signed_gate, "n_seqs": w.n_seqs, "tokens": w.tokens,
            "seq_lens": "16 x U{512..8192} (seed 0) + 65536", "io_dtype": w.io_dtype,
            "o_dtype": w.o_dtype, "state_dtype": "f32", "S0": "N(0, 0.02) per sequence",
            "l2": "inputs larger than L2 (q,k,v,a 4.4 GB + o 1.1 GB per step)"}


def to_dev(host, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in host.items()}


class PrefillCase:
    """One workload's device buffers and its ckda_chunk_fwd call."""

    def __init__(self, ops, w, host, dev, signed_gate=None):
        self.ops, self.w = ops, w
        self.sg = w.signed_gate if signed_gate is None else signed_gate
        self.d = to_dev(host, dev)
        B, T = host["q"].shape[:2]
        self.o = torch.empty((B, T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
        self.S_T = torch.empty((w.n_seqs, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        self.ws = ops.new_workspace(B, T, w.H, w.dk, w.dv, w.chunk,
                                    w.n_seqs if w.seq_lens is not None else 0, dev)

    def __call__(self):
        d = self.d
        self.ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["S0"], d["cu_seqlens"],
                           chunk=self.w.chunk, signed_gate=self.sg, o=self.o, S_T=self.S_T,
                           workspace=self.ws)

    def check(self, what):
        st = self.ops.workspace_status(self.ws)
        if st != 0:
            raise RuntimeError(f"device status {st} after {what}")

    def plan(self):
        """What the unit planner decided in the last call (the plan's header at byte 128 of the
        workspace: units of the two launches per head, sequences cut, segments of each), or
        None for an unplanned call (unpacked without a cut: the header stays zero)."""
        if self.ws.numel() < 176:
            return None
        h = self.ws[128:176].view(torch.int32).cpu().tolist()
        n1, n3, nsplit = h[0], h[1], h[2]
        if n1 == 0 and n3 == 0:
            return None
        return {"cut_sequences": nsplit, "segments": [h[4 + 4 * i] for i in range(nsplit)],
                "first_launch_units": n1 * self.w.H, "second_launch_units": n3 * self.w.H}


def prefill_roofline(w, ms_launch, peaks, traffic_key):
    byts = prefill_bytes(w)
    flops = prefill_flops_per_token_head(w.dk, w.dv, w.chunk) * w.tokens * w.H
    gbs = byts / (ms_launch * 1e-3) / 1e9
    tf = flops / (ms_launch * 1e-3) / 1e12
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "traffic": profiled_traffic(traffic_key),
            "peak_source": peaks["source"], "algorithmic_bytes_per_launch": byts,
            "algorithmic_flop_per_launch": flops, "tensor_tflops": tf,
            "tensor_frac_of_bf16": tf / peaks["bf16_tflops"]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ckda", choices=["ckda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="timed decode steps (default: --steps rounded up to the 128-step cycle)")
    ap.add_argument("--legs", default="varlen,e2e,kda,spread,fast,ratio,bwd,decode",
                    help="comma list of legs to run (varlen = the headline, e2e, kda, spread, "
                         "fast = KDA with fast-forgetting channels, ratio, bwd, decode); a "
                         "profiling run can select one, the default runs all")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    from linear_rnn_ckda_b200 import ops

    ops.load()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    legs = set(args.legs.split(","))
    extra_steps = max(3, min(args.steps, 10))

    # ------------------------------------------------------------ headline: varlen CKDA
    # (a profiling run that leaves the headline out of --legs skips it and its e2e leg)
    w = HEADLINE
    run_head = "varlen" in legs
    tokens = w.tokens * world
    ms = ms_step = value = float("nan")
    roofline = head_plan = None
    host = case = None
    clk = ClockSampler(local)
    if run_head:
        host = synth.make_prefill(w, seed=rank)
        case = PrefillCase(ops, w, host, dev)
        with clk:
            ms = time_loop(case, args.steps, args.warmup, world, stream)
        ms = max_over_ranks(ms, world)
        case.check("the headline leg")
        head_plan = case.plan()
        ms_step = ms / args.steps
        value = tokens * args.steps / (ms / 1000.0)
        # dominant kernel: the chunk kernel.  A packed step is six launches (the 256-byte status
        # memset before them is included, < 2 us): the unit planner, the first launch of the
        # plain tensor-core kernel and of the kernel with per-channel references for the units
        # it handed off (none here: its CTAs return at once, ~6 us with the programmatic
        # dependent launch), the state chain of the cut sequence, and the second pair; an
        # unpacked step without a cut is the first pair alone
        roofline = prefill_roofline(w, ms_step, peaks, "chunk_tc_kernel/" + w.name)

    # ------------------------------------------------------------ e2e (host buffers)
    # Each step copies its own q, k, v, a, b, S0 and cu_seqlens from pinned host memory, runs
    # ckda_chunk_fwd and reads o and S_T back.  Steps are pipelined the way a streaming caller
    # would run them: input copies, compute and output copies on three streams with two sets
    # of device buffers, so one step's read-back overlaps the next step's upload.  Timed with
    # CUDA events from the first upload to the last read-back.
    e2e = None
    if run_head and "e2e" in legs:
        keys = [k for k in ("q", "k", "v", "a", "b", "S0", "cu_seqlens") if host.get(k) is not None]
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = case.o.numel() * case.o.element_size() + case.S_T.numel() * case.S_T.element_size()
        pin = {k: host[k].pin_memory() for k in keys}
        nbuf = 2
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        dd = [{k: torch.empty_like(host[k], device=dev) for k in keys} for _ in range(nbuf)]
        oo = [torch.empty_like(case.o) for _ in range(nbuf)]
        SS = [torch.empty_like(case.S_T) for _ in range(nbuf)]
        o_host = [torch.empty(case.o.shape, dtype=case.o.dtype).pin_memory() for _ in range(nbuf)]
        S_host = [torch.empty(case.S_T.shape, dtype=case.S_T.dtype).pin_memory()
                  for _ in range(nbuf)]
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_done = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]
        for e in ev_done + ev_out:
            e.record(stream)
        step_no = [0]

        def e2e_step():
            i = step_no[0] % nbuf
            step_no[0] += 1
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_done[i])          # the step that last used buffer set i
                for k in keys:
                    dd[i][k].copy_(pin[k], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])             # its outputs have been read back
            x = dd[i]
            ops.chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x.get("S0"), x.get("cu_seqlens"),
                          chunk=w.chunk, signed_gate=w.signed_gate, o=oo[i], S_T=SS[i],
                          workspace=case.ws)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                o_host[i].copy_(oo[i], non_blocking=True)
                S_host[i].copy_(SS[i], non_blocking=True)
                ev_out[i].record(s_out)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        t0e = torch.cuda.Event(enable_timing=True)
        t1e = torch.cuda.Event(enable_timing=True)
        t0e.record(s_in)
        for _ in range(extra_steps):
            e2e_step()
        s_in.wait_stream(stream)
        s_in.wait_stream(s_out)
        t1e.record(s_in)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(t0e.elapsed_time(t1e), world)
        case.check("the end-to-end leg")
        e2e = {"value": tokens * extra_steps / (ms_e2e / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ms_e2e / extra_steps, "steps": extra_steps,
               "pipelined": "2 buffer sets, 3 streams"}
        del dd, oo, SS, o_host, S_host, pin

    # ------------------------------------------------------------ CPU baseline (oracle)
    cpu = None
    if run_head and rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, cores, desc = cpu_baseline_sample(host, w, range(0, 16))
        cpu = {"value": v_cpu, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc}
    del case, host

    # ------------------------------------------------------------ the other prefill workloads
    workloads = {}
    for leg, wk in (("kda", KDA), ("spread", SPREAD), ("fast", synth.KDA_FAST)):
        if leg not in legs:
            continue
        c = PrefillCase(ops, wk, synth.make_prefill(wk, seed=rank), dev)
        ms_k = max_over_ranks(time_loop(c, extra_steps, args.warmup, world, stream), world)
        c.check(f"the {leg} leg")
        ms_l = ms_k / extra_steps
        workloads[wk.name] = {
            "ms_per_step": ms_l, "steps": extra_steps,
            "tokens_per_s": wk.tokens * world / (ms_l / 1000.0),
            "roofline": prefill_roofline(wk, ms_l, peaks, "chunk_tc_kernel/" + wk.name)}
        if leg == "kda" and "ratio" in legs:
            # the same kernel in signed-gate (CKDA) mode on the KDA shapes and inputs: the
            # throughput ratio the pages quote (96-97 %, forward and backward, on H100)
            c.sg = 1
            ms_c = max_over_ranks(time_loop(c, extra_steps, args.warmup, world, stream), world)
            c.check("the CKDA ratio leg")
            c.sg = wk.signed_gate
            ms_k2 = max_over_ranks(time_loop(c, extra_steps, args.warmup, world, stream), world)
            workloads[wk.name]["ckda_over_kda_throughput"] = (ms_k2 / extra_steps) / (
                ms_c / extra_steps)
            workloads[wk.name]["ckda_mode_ms_per_step"] = ms_c / extra_steps
        del c

    # ------------------------------------------------------------ forward + backward
    # The pages' kernel measurement is forward plus backward (CKDA at 96-97 % of KDA on H100):
    # one ckda_chunk_fwd and one ckda_chunk_bwd per step on the KDA workload's shapes and
    # inputs, in KDA mode and in CKDA mode (the same kernels, signed gates).
    fwd_bwd = None
    if "bwd" in legs:
        wk = KDA
        c = PrefillCase(ops, wk, synth.make_prefill(wk, seed=rank), dev)
        g = torch.Generator(device="cpu").manual_seed(1234 + rank)
        dO = torch.randn(c.o.shape, generator=g).to(device=dev, dtype=torch.bfloat16)
        bws = torch.empty(ops.bwd_workspace_size(wk.B, wk.T, wk.H, wk.dk, wk.dv, 0),
                          dtype=torch.uint8, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        grads = (torch.empty(c.d["q"].shape, **f32), torch.empty(c.d["k"].shape, **f32),
                 torch.empty(c.d["v"].shape, **f32), torch.empty(c.d["a"].shape, **f32),
                 torch.empty(c.d["b"].shape, **f32), None)
        res = {}
        for mode, sg in (("kda", 0), ("ckda", 1)):
            def fb():
                c.sg = sg
                c()
                ops.chunk_bwd(c.d["q"], c.d["k"], c.d["v"], c.d["a"], c.d["b"], None, None, dO=dO,
                              signed_gate=sg, want_dS0=False, workspace=bws, grads=grads)

            ms_fb = max_over_ranks(time_loop(fb, extra_steps, args.warmup, world, stream), world)
            if ops.workspace_status(bws) != 0:
                raise RuntimeError("device status after the backward leg")
            res[mode] = ms_fb / extra_steps
        c.sg = wk.signed_gate
        fwd_bwd = {"workload": wk.name, "steps": extra_steps,
                   "kda_ms_per_step": res["kda"], "ckda_ms_per_step": res["ckda"],
                   "kda_tokens_per_s": wk.tokens * world / (res["kda"] / 1000.0),
                   "ckda_over_kda_throughput": res["kda"] / res["ckda"],
                   "path": "forward: tcgen05 kernel; backward: exact fp32 CUDA-core kernels"}
        del c, grads, bws, dO

    # ------------------------------------------------------------ decode
    wd = DECODE
    dsteps = args.decode_steps or max(args.steps, 128)
    decode_obj = None
    if "decode" in legs:
        dq = {k: v.to(dev) for k, v in synth.make_decode(wd, seed=rank).items()}
        S = dq["S"]
        o_dec = torch.empty((wd.B, wd.H, wd.dv), dtype=torch.float32, device=dev)
        counter = [0]

        def decode():
            t = counter[0] % wd.decode_steps
            counter[0] += 1
            ops.decode_step(dq["q"][t], dq["k"][t], dq["v"][t], dq["a"][t], dq["b"][t], S,
                            signed_gate=wd.signed_gate, o_dtype=torch.float32, o=o_dec)

        ms_d = max_over_ranks(time_loop(decode, dsteps, args.warmup, world, stream), world)
        dbytes = decode_bytes(wd)
        dec_gbs = dbytes * world * dsteps / (ms_d / 1000.0) / 1e9
        decode_obj = {"value": dec_gbs, "unit": "GB/s", "frac": dec_gbs / world / peaks["hbm_gbs"],
                      "peak": peaks["hbm_gbs"], "ms_per_step": ms_d / dsteps, "steps": dsteps,
                      "workload": wd.name, "algorithmic_bytes_per_step": dbytes,
                      "state_bytes_per_step": wd.B * wd.H * wd.dk * wd.dv * 8,
                      "traffic": profiled_traffic("decode_kernel/" + wd.name)}

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; same shapes and distributions as the pages' workloads)",
            "config": headline_config(w),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "plan": head_plan,
            "workloads": workloads, "fwd_bwd": fwd_bwd, "decode": decode_obj,
            "gpu_launches": (6 if w.seq_lens is not None else 2) * args.steps, "clocks": clocks, "peaks_source": peaks["source"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
