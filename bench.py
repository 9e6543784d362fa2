#!/usr/bin/env python
"""Benchmark of the KDA chunked forward (libkda.so) on B200; prints ONE JSON line.

    python bench.py [--gpus N --steps K --warmup W] [--workload prefill_1m]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed on host cores

A step is one kda_fwd call over the whole workload (default: the 1M-token
prefill, B=1, H=8, T=2^20, d_k=d_v=128, bf16 q/k/v, fp32 gates, chunk 64).
``value`` is Mtokens/s with inputs resident in HBM (tokens counted once, not per
head); ``e2e`` is the same metric through the host-buffer entry point
kda_fwd_host with the host->device copy of the inputs and the device->host copy
of the outputs inside every timed step.  The workload's inputs (12.9 GB) are
larger than the 126 MB L2, so no flush is needed between steps.

``--workload decode_1024x1`` / ``verify_512x4`` time instead one decode /
multi-token verify step (kda_decode) over 1024 sequences x 1 token or 512
sequences x 4 tokens whose states (8 heads x 64 KiB each) stay resident and are
updated in place; there ``e2e`` copies the step's tokens up and its outputs back
through the Python binding while the states stay on the device.

With N GPUs (torchrun, one rank per GPU) every rank runs its own copy of the
workload (independent problems, no data-path collective): weak scaling, value =
N * tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_139_b200.inputs import (WORKLOADS, algorithmic_bytes,  # noqa: E402
                                              algorithmic_flops, is_decode, make_inputs,
                                              workload)

METRIC = "KDA chunked prefill Mtokens/s on 1 B200; % of bf16 tensor / HBM roofline"
METRIC_DECODE = "KDA decode/verify step Mtokens/s on 1 B200 (resident states); % of HBM roofline"
UNIT = "Mtokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(inp, n_gpus):
    return {"workload": inp.name, "B": inp.B, "T": inp.T, "H": inp.H, "d_k": inp.dk,
            "d_v": inp.dv, "chunk": inp.chunk, "num_seqs": inp.n_seqs,
            "tokens_per_gpu": inp.tokens, "qkv_dtype": "bf16" if inp.bf16 else "f32",
            "gates": "fp32 log_alpha, fp32 beta", "state": "fp32",
            "l2": "inputs larger than L2 (%.1f GB per step vs 126 MB L2), no flush" %
                  (algorithmic_bytes(inp) / 1e9),
            "parallelism": f"dp{n_gpus} (independent problem per GPU)"}


def decode_config(inp, n_gpus):
    st = inp.n_seqs * inp.H * inp.dk * inp.dv * 4
    return {"workload": inp.name, "step": "decode/verify on resident states (kda_decode)",
            "sequences": inp.B, "new_tokens_per_seq": inp.T, "H": inp.H, "d_k": inp.dk,
            "d_v": inp.dv, "tokens_per_gpu": inp.tokens,
            "qkv_dtype": "bf16" if inp.bf16 else "f32", "gates": "fp32 log_alpha, fp32 beta",
            "state": "fp32, updated in place",
            "l2": "states larger than L2 (%.0f MB vs 126 MB L2), no flush" % (st / 1e6),
            "parallelism": f"dp{n_gpus} (independent problem per GPU)"}


# ------------------------------------------------------------------ multi-rank helpers
def max_over_ranks(ms: float, dist_mod=None, device=None) -> float:
    """Slowest rank's time (every rank calls this at the same point)."""
    if dist_mod is None or not dist_mod.is_initialized() or dist_mod.get_world_size() == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, ms: float) -> float:
    """Whole-job Mtokens/s: every rank processes its own problem of tokens_per_rank
    tokens; the job takes as long as its slowest rank."""
    return world * tokens_per_rank / (ms * 1e-3) / 1e6


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms) of one GPU while the timed region runs."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"kda_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0]:
                continue
            rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(
                    (float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------ oracle baseline
def decode_sample(name: str, target_s: float, seed: int = 0):
    """Sequences of a decode workload's recipe that take the oracle about
    target_s seconds (whole workload at most): (inputs, threads)."""
    import oracle
    spec = dict(WORKLOADS[name])
    spec.pop("step")
    B = spec.pop("B")
    threads = min(len(os.sched_getaffinity(0)), spec["H"])
    probe = make_inputs(B=min(B, 32), seed=seed, name=name, **spec)
    t0 = time.perf_counter()
    oracle.recurrent(probe.q, probe.k, probe.v, probe.log_alpha, probe.beta,
                     probe.initial_state, None, threads=threads)
    per_seq = max(time.perf_counter() - t0, 1e-6) / probe.B
    n = int(max(1, min(B, target_s / per_seq)))
    return make_inputs(B=n, seed=seed, name=name, **spec), threads


def oracle_sample_rate(inp_name: str, target_s: float = 15.0, seed: int = 0):
    """Time the fp64 oracle on a bounded prefix of the workload's recipe."""
    import oracle
    if is_decode(inp_name):
        x, threads = decode_sample(inp_name, target_s, seed)
        t0 = time.perf_counter()
        oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, None,
                         threads=threads)
        dt = time.perf_counter() - t0
        return {"value": x.tokens / dt / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
                "sample": f"{x.B} of the sequences x {x.T} tokens x {x.H} heads of the "
                          f"{inp_name} recipe (fp64 token recurrence, {dt:.1f} s)",
                "seconds": dt}
    spec = dict(WORKLOADS[inp_name])
    spec.pop("packed", None)
    spec.pop("T", None)
    H = spec["H"]
    probe_T = 1024
    x = make_inputs(T=probe_T, seed=seed, name=inp_name, **{k: v for k, v in spec.items()
                                                              if k != "B"}, B=1)
    t0 = time.perf_counter()
    oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, None, o_tokens=0)
    rate = probe_T / max(time.perf_counter() - t0, 1e-6)  # tokens/s (all heads)
    T_s = int(max(probe_T, min(rate * target_s, 1 << 20)))
    T_s = (T_s // 64) * 64
    x = make_inputs(T=T_s, seed=seed, name=inp_name, **{k: v for k, v in spec.items()
                                                          if k != "B"}, B=1)
    threads = min(len(os.sched_getaffinity(0)), H)
    t0 = time.perf_counter()
    oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, None, o_tokens=0,
                     threads=threads)
    dt = time.perf_counter() - t0
    return {"value": T_s / dt / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"first {T_s} tokens x {H} heads of the {inp_name} recipe "
                      f"(fp64 token recurrence, {dt:.1f} s)", "seconds": dt}


def run_reference(args, rank, world):
    """The oracle as it stands, on host cores: rank 0 only."""
    if rank != 0:
        return
    import oracle
    name = args.workload
    if is_decode(name):
        return run_reference_decode(args, world)
    spec = dict(WORKLOADS[name])
    spec.pop("packed", None)
    spec.pop("T", None)
    spec.pop("B", None)
    H = spec["H"]
    threads = min(len(os.sched_getaffinity(0)), H)
    # size each step to ~2 s of oracle work
    probe = make_inputs(B=1, T=512, seed=0, name=name, **spec)
    t0 = time.perf_counter()
    oracle.recurrent(probe.q, probe.k, probe.v, probe.log_alpha, probe.beta, None, None,
                     o_tokens=0, threads=threads)
    rate = 512 / max(time.perf_counter() - t0, 1e-6)
    T_s = max(64, int(rate * 2.0) // 64 * 64)
    x = make_inputs(B=1, T=T_s, seed=0, name=name, **spec)
    f = lambda: oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, None,
                                 o_tokens=T_s, threads=threads)
    for _ in range(args.warmup):
        f()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        f()
        times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    val = T_s / step / 1e6
    full = workload_config(x, world)
    full.update({"workload": name, "T": None, "sampled_T": T_s})
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": full,
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"first {T_s} tokens x {H} heads of the {name} recipe "
                                       "per step (fp64 token recurrence)"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_decode(args, world):
    import oracle
    x, threads = decode_sample(args.workload, 2.0)
    f = lambda: oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state, None,
                                 threads=threads)
    for _ in range(args.warmup):
        f()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        f()
        times.append(time.perf_counter() - t0)
    step = sum(times) / len(times)
    val = x.tokens / step / 1e6
    cfg = decode_config(x, world)
    cfg["sampled_sequences"] = x.B
    sample = (f"{x.B} of the sequences x {x.T} tokens x {x.H} heads of the {args.workload} "
              "recipe per step (fp64 token recurrence)")
    line = {"impl": "reference", "metric": METRIC_DECODE, "value": val, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ per-kernel bytes
def segment_plan(inp, sms=148):
    """Segment length (chunks) the library picks for this workload (same rule as
    the host planner in kda_api.cu), and whether sequences are cut."""
    C = 64
    nch_max = (inp.T + C - 1) // C
    target = 2 * sms
    if inp.cu_seqlens is None:
        G = max(1, round(target / (inp.B * inp.H)))
        seg = (nch_max + G - 1) // G
    else:
        nch_total = nch_max + inp.n_seqs
        seg = (nch_total * inp.H + target - 1) // target
    seg = max(seg, 8)
    return seg, seg < nch_max


def kernel_algorithmic_bytes(name, inp, path_bytes):
    """Minimum bytes one launch of kernel `name` must move for what it computes.

    pass 3 (forward) delivers the path's results from its inputs: the whole
    path's algorithmic bytes.  Pass 1 (segment transitions and chunk operands),
    run when the plan cuts a sequence, builds every chunk's operands for pass 3
    and the transition of every segment that has a successor: it must read q, k,
    v, log alpha and beta of every token once and write one (B, M) pair
    (2 x 128 x 128 fp32) per such segment and head.  The chunk cache it leaves
    for pass 3 is an intermediate of this design and is not counted: it shows up
    in the measured DRAM traffic instead."""
    if name != "tc_pass1_transitions":
        return path_bytes
    seg, cut = segment_plan(inp)
    if not cut:
        return 0
    per_tok = inp.H * (inp.dk * 2 * 2 + inp.dv * 2 + inp.dk * 4 + 4)
    toks = segs = 0
    for L in inp.seq_lens:
        L = int(L)
        nch = (L + 63) // 64
        g = max(1, (nch + seg - 1) // seg)
        segs += g - 1
        toks += L
    return toks * per_tok + segs * inp.H * 2 * inp.dk * inp.dv * 4


# ------------------------------------------------------------------ traffic record
def recorded_traffic(kernel_tag: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it is for this
    workload and its kernel sources are unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel_tag)
    if not rec or rec.get("workload") != workload_name:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return rec["bytes_per_launch"] if h.hexdigest() == rec["sha256"] else None


# ------------------------------------------------------------------ context parallel, emulated
def run_cp_emulation(args):
    """Each of W virtual ranks owns T/W tokens of every sequence.  Rank r runs
    kda_span_transition on its span, kda_apply_transitions on the transitions of
    ranks < r (the all-gather's result), then kda_span_forward from that state
    (which reuses the transition's per-segment work).  On one
    GPU the ranks run one after another; each rank's work is timed with CUDA
    events, and a W-GPU run would take the slowest rank's time plus one
    all-gather of W x B x H x 128 KiB (estimated here at the measured 770 GB/s
    NVLink peer bandwidth, never timed)."""
    import torch
    import gated_delta_rule_139_b200 as kda

    W = args.cp_emulate
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = workload(args.workload, seed=0)
    if inp.cu_seqlens is not None or inp.T % W or not inp.bf16 or inp.dk != 128:
        raise SystemExit("--cp-emulate needs an unpacked bf16 d=128 workload with T divisible by W")
    span = inp.T // W
    t = lambda a: torch.from_numpy(a).view(torch.bfloat16) if a.dtype == np.uint16 else \
        torch.from_numpy(a)
    full = {k_: t(getattr(inp, k_)).to(dev) for k_ in ("q", "k", "v", "log_alpha", "beta")}
    s0 = None if inp.initial_state is None else torch.from_numpy(inp.initial_state).to(dev)
    spans = [{k_: full[k_][:, r * span:(r + 1) * span].contiguous() for k_ in full}
             for r in range(W)]
    del full
    stream = torch.cuda.current_stream(dev)
    ws = [kda.span_workspace(s["k"]) for s in spans]
    trans = [kda.kda_span_transition(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], w)
             for s, w in zip(spans, ws)]
    gathered = torch.stack(trans)

    def rank_step(r):  # transition (kept work in ws[r]), incoming state, forward
        s = spans[r]
        kda.kda_span_transition(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], ws[r],
                                out=trans[r])
        s_in = kda.kda_apply_transitions(gathered[:r], s0)
        return kda.kda_span_forward(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], ws[r], s_in)

    per_rank = []
    for r in range(W):
        for _ in range(args.warmup):
            rank_step(r)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            rank_step(r)
        e1.record(stream)
        torch.cuda.synchronize()
        per_rank.append(e0.elapsed_time(e1) / args.steps)
    gather_bytes = W * inp.B * inp.H * 2 * 128 * 128 * 4
    gather_ms = gather_bytes / 770e9 * 1e3
    proj_ms = max(per_rank) + gather_ms
    tokens = inp.tokens
    line = {"metric": METRIC + " -- context parallel, emulated", "value": tokens / (proj_ms * 1e-3) / 1e6,
            "unit": UNIT, "n_gpus": 1, "emulated_ranks": W, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": proj_ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(inp, 1), parallelism=f"cp{W} emulated on 1 GPU",
                           span_tokens=span),
            "per_rank_ms": per_rank, "sum_of_ranks_ms": sum(per_rank),
            "allgather": {"bytes": gather_bytes, "ms_estimate": gather_ms,
                          "basis": "770 GB/s measured NVLink peer copy; not timed"},
            "note": "ms_per_step = slowest emulated rank + all-gather estimate"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_1m", choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer measurement")
    ap.add_argument("--out-gate", action="store_true",
                    help="fuse an output gate (random values in (0, 1), dtype of q) into the "
                         "step (kda_fwd_ex / kda_decode)")
    ap.add_argument("--cp-emulate", type=int, default=0, metavar="W",
                    help="context-parallel prefill of the workload over W ranks, emulated on "
                         "one GPU: the ranks' span work runs one after another and is timed "
                         "per rank (not a multi-GPU measurement)")
    ap.add_argument("--snap-interval", type=int, default=0,
                    help="forward workloads: also write a prefix-cache state snapshot every "
                         "this many tokens (kda_fwd_snap), each to its own pool row")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.cp_emulate:
        run_cp_emulation(args)
        return

    import torch
    import gated_delta_rule_139_b200 as kda

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist

    inp = workload(args.workload, seed=rank)
    tokens = inp.tokens
    bf16 = inp.bf16

    # pinned host copies (for e2e) and device-resident copies (for value)
    def pinned(a):
        t = torch.from_numpy(a)
        if bf16 and a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.pin_memory()

    host = {k: (None if getattr(inp, k) is None else pinned(getattr(inp, k)))
            for k in ("q", "k", "v", "log_alpha", "beta", "initial_state")}
    alg_bytes = algorithmic_bytes(inp)
    # a decode token costs 7 flops per state element (decay; S^T k; rank-1 update; S^T q)
    alg_flops = (7.0 * inp.tokens * inp.H * inp.dk * inp.dv if is_decode(args.workload)
                 else algorithmic_flops(inp))
    v_shape = tuple(inp.v.shape)
    for k_ in ("q", "k", "v", "log_alpha", "beta"):
        setattr(inp, k_, None)  # the pinned copies are the host data from here on
    cu_host = inp.cu_seqlens
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        d = {k: (None if t is None else t.to(dev, non_blocking=True)) for k, t in host.items()}
        cu_dev = None if cu_host is None else torch.from_numpy(cu_host).to(dev)
        out = torch.empty(v_shape, dtype=d["q"].dtype, device=dev)
        fs = torch.empty((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=torch.float32, device=dev)
    stream.synchronize()

    decode = is_decode(args.workload)
    snap = None
    if args.snap_interval and not decode:
        lens = [int(x) for x in inp.seq_lens]
        max_snaps = max(1, max(lens) // args.snap_interval)
        n_snaps = sum(L // args.snap_interval for L in lens)
        with torch.cuda.stream(stream):
            slots = torch.arange(inp.n_seqs * max_snaps, dtype=torch.int32,
                                 device=dev).reshape(inp.n_seqs, max_snaps)
            pool = torch.empty((inp.n_seqs * max_snaps, inp.H, inp.dk, inp.dv),
                               dtype=torch.float32, device=dev)
        snap = {"slots": slots, "pool": pool, "count": n_snaps}
        alg_bytes += n_snaps * inp.H * inp.dk * inp.dv * 4

    gate = None
    if args.out_gate:
        with torch.cuda.stream(stream):
            g = torch.Generator(device=dev)
            g.manual_seed(1000 + rank)
            gate = torch.rand(v_shape, generator=g, device=dev).to(d["q"].dtype)
        alg_bytes += gate.numel() * gate.element_size()

    def step():
        if decode:  # the state is updated in place, step after step
            kda.kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], out=out, stream=stream, out_gate=gate)
        elif snap is not None:
            kda.kda_fwd_snap(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                             d["initial_state"], cu_dev, snap_interval=args.snap_interval,
                             snap_slots=snap["slots"], snap_pool=snap["pool"], out=out,
                             final_state=fs, stream=stream, out_gate=gate)
        else:
            kda.kda_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"],
                        cu_dev, 64, out, fs, stream=stream, out_gate=gate)
        return kda.last_launch_count()

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    launches = 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the headline: K steps with no per-launch instrumentation
    with ClockSampler(uuid) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            launches += step()
        ev1.record(stream)
        stream.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, pg, dev)
    # a second, separate loop with CUDA events around every internal launch (on the
    # stream the kernels run on) for the per-kernel times and shares
    kda.profile_read()  # discard earlier records
    kda.profile_enable(True)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        step()
    p1.record(stream)
    stream.synchronize()
    kda.profile_enable(False)
    per_kernel = kda.profile_read()
    prof_ms = p0.elapsed_time(p1) / args.steps
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    clocks = clk.summary()
    value = job_throughput(world, tokens, ms)

    # e2e: host buffers through kda_fwd_host, copies inside every step
    nbytes = lambda t: 0 if t is None else t.numel() * t.element_size()
    e2e = None
    if not args.no_e2e and snap is None and gate is None:
        out_h = torch.empty(v_shape, dtype=host["q"].dtype).pin_memory()
        fs_h = torch.empty((inp.n_seqs, inp.H, inp.dk, inp.dv), dtype=torch.float32).pin_memory()
        cu_arg = None if cu_host is None else np.ascontiguousarray(cu_host, dtype=np.int32)

        tok_keys = ("q", "k", "v", "log_alpha", "beta")

        def e2e_step():
            if decode:
                # a serving step: this step's tokens go up, the outputs come back,
                # the states stay resident on the device
                with torch.cuda.stream(stream):
                    x = {k_: host[k_].to(dev, non_blocking=True) for k_ in tok_keys}
                    o, _ = kda.kda_decode(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                          d["initial_state"], stream=stream)
                    out_h.copy_(o, non_blocking=True)
            else:
                kda.kda_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"],
                                 host["beta"], host["initial_state"], cu_arg, 64, out_h, fs_h,
                                 stream=stream)

        e2e_step()
        if pg:
            pg.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, pg, dev)
        if decode:
            h2d = sum(nbytes(host[k_]) for k_ in tok_keys)
            d2h = nbytes(out_h)
        else:
            h2d = sum(nbytes(t) for t in host.values()) + (0 if cu_arg is None else cu_arg.nbytes)
            d2h = nbytes(out_h) + nbytes(fs_h)
        e2e = {"value": job_throughput(world, tokens, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": args.e2e_steps}

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    cfg = decode_config(inp, world) if decode else workload_config(inp, world)
    if gate is not None:
        cfg["out_gate"] = "fused output gate, %s, shape of out" % str(gate.dtype).split(".")[-1]
    if snap is not None:
        cfg["snapshots"] = {"interval_tokens": args.snap_interval, "count": snap["count"],
                            "bytes": snap["count"] * inp.H * inp.dk * inp.dv * 4,
                            "entry": "kda_fwd_snap"}
    kernels = {name: {"ms_per_launch": tot / n, "launches": n,
                      "share": tot / (prof_ms * args.steps)}
               for name, (tot, n) in per_kernel.items()}
    dom = max(kernels, key=lambda k_: kernels[k_]["ms_per_launch"] * kernels[k_]["launches"])
    dom_bytes = kernel_algorithmic_bytes(dom, inp, alg_bytes)
    achieved = dom_bytes / (kernels[dom]["ms_per_launch"] * 1e-3) / 1e9
    t_roof = max(alg_bytes / (peaks["hbm_gbs"] * 1e9), alg_flops / (peaks["bf16_tflops"] * 1e12))
    line = {
        "metric": METRIC_DECODE if decode else METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if kda.last_path() in ("ffma", "decode") else "bf16",
        "data": "synthetic",
        "config": cfg,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic(dom, inp.name),
                     "kernel": dom,
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s",
                     "path": {"algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops,
                              "roofline_ms": t_roof * 1e3,
                              "frac_of_roofline": t_roof / (ms * 1e-3)},
                     "kernels": kernels},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample_rate(args.workload)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
