#!/usr/bin/env python3
"""Benchmark of the KDA / Complex-KDA hot path on B200.

Prints ONE JSON line (rank 0).  The headline is the chunkwise prefill
(``ckda_chunk_fwd``) on the standard KDA workload B=4, H=16, T=4096,
dk=dv=128, chunk 64, bf16 q/k/v/a, bf16 o, fp32 state: ``value`` is prefill
tokens/s for the whole job, one step = one ``ckda_chunk_fwd`` call over the
whole batch with its inputs resident in HBM.  The same run times the decode
step (``ckda_decode_step``, B=256, H=32, d=128, fp32 state updated in place,
bf16 q/k/v/a, fp32 o) and reports its state GB/s against HBM in ``decode``.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workload on
its own seeded data (independent (sequence, head) units, no data-path
collective); ``value`` = all ranks' tokens / max-over-ranks time ("weak").

``--impl reference`` times the fp64 CPU oracle (the only other arm; there is
no installable reference implementation) on a bounded sample of the same
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

PREFILL = synth.KDA_STD
DECODE = synth.DECODE
SPREAD = synth.CKDA_SPREAD

# Algorithmic counts per unit (d = dk = dv = 128, chunk C = 64):
#   prefill FLOP per token-head = 6 d^2 + C (3 dk + 2 dv) + C^2 / 3
#   prefill bytes per token-head = q + k + v + a (bf16) + b (fp32) + o (bf16)
#   plus S_T (fp32 d^2) per (sequence, head); S0 is not read (zero state)
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


def profiled_traffic(kernel):
    """DRAM bytes per launch from the committed ncu capture of `kernel`, or None
    when the kernel's sources changed after the capture."""
    try:
        with open(PROFILED) as f:
            rec = json.load(f)[kernel]
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


def cpu_oracle_sample(w, seed, max_units=None):
    """Oracle on a bounded sample of (sequence, head) units of workload w: (seconds, token-heads, cores)."""
    import numpy as np

    import oracle

    cores = os.cpu_count() or 1
    H = w.H
    inp = synth.make_prefill(w.with_(B=1), seed)  # one batch row = H units of T tokens
    units = H if max_units is None else min(H, max_units)
    f = lambda t: t[:, :, :units].to(torch.float64).numpy()
    q, k, v, a = (np.ascontiguousarray(f(inp[x])) for x in "qkva")
    b = np.ascontiguousarray(inp["b"][:, :, :units].to(torch.float64).numpy())
    oracle.build()
    t0 = time.perf_counter()
    oracle.ckda_fwd(q, k, v, a, b, None, signed_gate=w.signed_gate, threads=cores)
    dt = time.perf_counter() - t0
    return dt, units * w.T, min(cores, units)


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = PREFILL
    times = []
    th = 0
    cores = 1
    for i in range(args.warmup + args.steps):
        dt, th, cores = cpu_oracle_sample(w, seed=i)
        if i >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = (th / w.H) * len(times) / tot  # tokens/s (a token carries H heads)
    sample = f"one batch row of {w.name}: {w.H} heads x {w.T} tokens per step (fp64, sequential per head)"
    line = {
        "impl": "reference", "metric": "chunk-fwd prefill tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * tot / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ckda", choices=["ckda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="timed decode steps (default: --steps rounded up to the 128-step cycle)")
    ap.add_argument("--legs", default="prefill,e2e,ckda,decode",
                    help="comma list of legs to run (prefill, e2e, ckda, decode); a profiling "
                         "run can select one, the default runs all")
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
    # ------------------------------------------------------------ prefill leg
    w = PREFILL
    host = synth.make_prefill(w, seed=rank)
    d = {k: (None if v is None else v.to(dev)) for k, v in host.items()}
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((w.n_seqs, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    ws = ops.new_workspace(w.B, w.T, w.H, w.dk, w.dv, w.chunk, 0, dev)

    def prefill():
        ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], None, None, chunk=w.chunk,
                      signed_gate=w.signed_gate, o=o, S_T=S_T, workspace=ws)

    with ClockSampler(local) as clk:
        ms = time_loop(prefill, args.steps if "prefill" in legs else 1,
                       args.warmup if "prefill" in legs else 0, world, stream)
    if "prefill" not in legs:
        ms = float("nan")
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    tokens = w.tokens * world
    value = tokens * args.steps / (ms / 1000.0)
    status = ops.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the prefill leg")

    # dominant kernel: the chunk kernel; its launch average from the same events
    # (the memset of the 256-byte status word is included, < 2 us)
    byts = prefill_bytes(w)
    flops = prefill_flops_per_token_head(w.dk, w.dv, w.chunk) * w.tokens * w.H
    achieved_gbs = byts / (ms_step * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"],
                "traffic": profiled_traffic("chunk_tc_kernel"),
                "peak_source": peaks["source"],
                "algorithmic_bytes_per_launch": byts, "algorithmic_flop_per_launch": flops,
                "tensor_tflops": flops / (ms_step * 1e-3) / 1e12,
                "tensor_frac_of_bf16": flops / (ms_step * 1e-3) / 1e12 / peaks["bf16_tflops"]}

    # ------------------------------------------------------------ e2e prefill (host buffers)
    # Each step copies its own q, k, v, a, b from pinned host memory, runs ckda_chunk_fwd and
    # reads o and S_T back.  Steps are pipelined the way a streaming caller would run them:
    # input copies, compute and output copies on three streams with two sets of device
    # buffers, so one step's read-back overlaps the next step's upload (the link carries the
    # two directions at once).  Timed with CUDA events from the first upload to the last
    # read-back.
    e2e = None
    pin = {k: (None if v is None else v.pin_memory()) for k, v in host.items()}
    h2d = sum(v.numel() * v.element_size() for k, v in pin.items() if v is not None and k in "qkvab")
    d2h = o.numel() * o.element_size() + S_T.numel() * S_T.element_size()
    if "e2e" in legs:
        nbuf = 2
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        dd = [{k: torch.empty_like(host[k], device=dev) for k in "qkvab"} for _ in range(nbuf)]
        oo = [torch.empty_like(o) for _ in range(nbuf)]
        SS = [torch.empty_like(S_T) for _ in range(nbuf)]
        o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(nbuf)]
        S_host = [torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory() for _ in range(nbuf)]
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
                for k in "qkvab":
                    dd[i][k].copy_(pin[k], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])             # its outputs have been read back
            ops.chunk_fwd(dd[i]["q"], dd[i]["k"], dd[i]["v"], dd[i]["a"], dd[i]["b"], None, None,
                          chunk=w.chunk, signed_gate=w.signed_gate, o=oo[i], S_T=SS[i],
                          workspace=ws)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                o_host[i].copy_(oo[i], non_blocking=True)
                S_host[i].copy_(SS[i], non_blocking=True)
                ev_out[i].record(s_out)

        e2e_steps = max(3, min(args.steps, 10))
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        t0e = torch.cuda.Event(enable_timing=True)
        t1e = torch.cuda.Event(enable_timing=True)
        t0e.record(s_in)
        for _ in range(e2e_steps):
            e2e_step()
        s_in.wait_stream(stream)
        s_in.wait_stream(s_out)
        t1e.record(s_in)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(t0e.elapsed_time(t1e), world)
        if ops.workspace_status(ws) != 0:
            raise RuntimeError("device status after the end-to-end leg")
        e2e = {"value": tokens * e2e_steps / (ms_e2e / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ms_e2e / e2e_steps, "pipelined": "2 buffer sets, 3 streams"}
        del dd, oo, SS, o_host, S_host
    del pin

    # ------------------------------------------------------------ CKDA legs
    # the same kernel in signed-gate (CKDA) mode: on the KDA shapes and inputs (the throughput
    # ratio the pages quote as 96-97%), and on the CKDA spread-init workload
    ckda = None
    if "ckda" in legs:
        csteps = max(3, min(args.steps, 10))

        def prefill_ckda():
            ops.chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], None, None, chunk=w.chunk,
                          signed_gate=1, o=o, S_T=S_T, workspace=ws)

        ms_k = max_over_ranks(time_loop(prefill, csteps, args.warmup, world, stream), world)
        ms_c = max_over_ranks(time_loop(prefill_ckda, csteps, args.warmup, world, stream), world)
        if ops.workspace_status(ws) != 0:
            raise RuntimeError("device status after the CKDA leg")
        ws_ = SPREAD
        hs = synth.make_prefill(ws_, seed=rank)
        ds = {k: (None if v is None else v.to(dev)) for k, v in hs.items()}
        os_ = torch.empty((ws_.B, ws_.T, ws_.H, ws_.dv), dtype=torch.bfloat16, device=dev)
        Ss = torch.empty((ws_.n_seqs, ws_.H, ws_.dk, ws_.dv), dtype=torch.float32, device=dev)
        wss = ops.new_workspace(ws_.B, ws_.T, ws_.H, ws_.dk, ws_.dv, ws_.chunk, 0, dev)

        def spread():
            ops.chunk_fwd(ds["q"], ds["k"], ds["v"], ds["a"], ds["b"], ds["S0"], None,
                          chunk=ws_.chunk, signed_gate=ws_.signed_gate, o=os_, S_T=Ss,
                          workspace=wss)

        ms_s = max_over_ranks(time_loop(spread, csteps, args.warmup, world, stream), world)
        if ops.workspace_status(wss) != 0:
            raise RuntimeError("device status after the CKDA spread leg")
        ckda = {"workload": w.name, "steps": csteps,
                "kda_ms_per_step": ms_k / csteps, "ckda_ms_per_step": ms_c / csteps,
                "ckda_over_kda_throughput": ms_k / ms_c,
                "spread": {"workload": ws_.name, "ms_per_step": ms_s / csteps,
                           "tokens_per_s": ws_.tokens * world * csteps / (ms_s / 1000.0),
                           "hbm_gbs": prefill_bytes(ws_) * world * csteps / (ms_s / 1000.0) / 1e9}}
        del ds, os_, Ss, wss

    # ------------------------------------------------------------ decode leg
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
                      "traffic": profiled_traffic("decode_kernel")}

    # ------------------------------------------------------------ CPU baseline (oracle)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, th, cores = cpu_oracle_sample(w, seed=0)
        cpu = {"value": (th / w.H) / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"one batch row of {w.name} ({w.H} heads x {w.T} tokens), "
                         f"fp64 sequential per head, {dt:.2f} s wall"}

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": "chunk-fwd prefill tokens/s (+ % roofline); decode state GB/s vs HBM",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; same shapes and distributions as the pages' workloads)",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "chunk": w.chunk, "signed_gate": w.signed_gate, "io_dtype": w.io_dtype,
                       "o_dtype": w.o_dtype, "state_dtype": "f32",
                       "l2": "inputs larger than L2 (q,k,v,a 268 MB + o 67 MB per step)"},
            "roofline": roofline, "decode": decode_obj, "ckda": ckda, "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps, "clocks": clocks, "peaks_source": peaks["source"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
