"""Cycles per chunk of the transition pass, by phase, from the phase-trace build.

    python -m gated_delta_rule_139_b200.build --trace
    KDA_LIBRARY=_build/trace/libkda.so \\
        python -m gated_delta_rule_139_b200.phase_trace prefill_1m --first-chunk 300

The trace build (-DKDA_PHASE_TRACE) records, for CTA (0, 0) of the tensor-core
kernels, the SM clock at the phase boundaries of 64 consecutive chunks starting at
--first-chunk (prep warps and chain warps separately), and for every CTA of the
transition pass (pass 1) its start and end on the global timer, its SM, its chunk
count and its SM clock at both ends.  This runs kda_fwd three times on the named
workload and prints, from the last call: the CTA and SM spread of pass 1, the SM
clock it ran at, and the median cycles each phase of a chunk takes.
"""
from __future__ import annotations

import argparse
import ctypes

import numpy as np

PREP = {14: "raw tiles landed", 1: "gate prefix sums", 2: "operand images", 3: "[A;P] product",
        8: "inv: A from TMEM", 9: "inv: diagonal blocks", 10: "inv: T_21 in halves",
        11: "inv: barrier", 12: "inv: Z = A_21 T_lo", 4: "inv: T_hi Z into TB",
        5: "slot handed to the chain"}
CHAIN_TRANS = {1: "slot full", 2: "W, U' products, W image, B staged", 3: "B: U product", 4: "B: U staged",
               5: "M: state staged", 6: "M: U product", 7: "M: U staged"}


def _phases(st, names, label):
    valid = [c for c in range(1, 62) if st[c, 0] > 0 and st[c + 1, 0] > 0]
    if not valid:
        print(f"{label}: no chunks recorded")
        return
    per = np.array([st[c + 1, 0] - st[c, 0] for c in valid])
    ks = [k for k in names if all(st[c, k] > 0 for c in valid)]
    rel = {k: float(np.median([st[c, k] - st[c, 0] for c in valid])) for k in ks}
    ks.sort(key=lambda k: rel[k])
    print(f"{label}: {len(valid)} chunks, median {np.median(per):.0f} cycles per chunk")
    print(f"  {'phase (ends at)':24s} {'at':>7s} {'takes':>7s}")
    prev = 0.0
    for k in ks:
        print(f"  {names[k]:24s} {rel[k]:7.0f} {rel[k] - prev:7.0f}")
        prev = rel[k]
    print(f"  {'next chunk':24s} {np.median(per):7.0f} {np.median(per) - prev:7.0f}")


def main(argv=None) -> None:
    import torch

    import gated_delta_rule_139_b200 as kda
    from gated_delta_rule_139_b200.inputs import workload

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("workload")
    ap.add_argument("--first-chunk", type=int, default=2)
    args = ap.parse_args(argv)
    lib = kda.load_library()
    if not hasattr(lib, "kda_trace_spans"):
        raise SystemExit("not a trace build: set KDA_LIBRARY to _build/trace/libkda.so")
    lib.kda_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.kda_trace_spans.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.kda_trace_first_chunk.argtypes = [ctypes.c_longlong]
    if lib.kda_trace_first_chunk(args.first_chunk) != 0:
        raise SystemExit("kda_trace_first_chunk failed")
    inp = workload(args.workload, seed=0)
    dev = torch.device("cuda", 0)
    t = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)
    f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q, k, v = t(inp.q), t(inp.k), t(inp.v)
    la, be, s0, cu = f(inp.log_alpha), f(inp.beta), f(inp.initial_state), f(inp.cu_seqlens)
    for _ in range(3):
        kda.kda_fwd(q, k, v, la, be, s0, cu)
        torch.cuda.synchronize(dev)
    kda.check_device()

    sp = np.zeros((8192, 6), dtype=np.uint64)
    if lib.kda_trace_spans(sp.ctypes.data, sp.size) != sp.size:
        raise SystemExit("kda_trace_spans failed")
    sp = sp.astype(np.int64)
    s = sp[sp[:, 1] > sp[:, 0]]
    if len(s):
        t0 = s[:, 0].min()
        dur = (s[:, 1] - s[:, 0]) / 1e3
        per_sm = np.bincount(s[:, 2].astype(np.int64))
        mhz = (s[:, 5] - s[:, 4]) / (s[:, 1] - s[:, 0]) * 1e3
        print(f"{args.workload}: pass 1 CTAs {len(s)} on {np.count_nonzero(per_sm)} SMs "
              f"(at most {per_sm.max()} per SM), span {(s[:, 1].max() - t0) / 1e3:.1f} us")
        print(f"  CTA time us: min {dur.min():.1f} median {np.median(dur):.1f} max {dur.max():.1f}; "
              f"chunks per CTA median {np.median(s[:, 3]):.0f}; "
              f"ns per chunk median {np.median(dur * 1e3 / np.maximum(s[:, 3], 1)):.0f}")
        print(f"  SM clock over a CTA (MHz): min {mhz.min():.0f} median {np.median(mhz):.0f} "
              f"max {mhz.max():.0f}")
    buf = np.zeros((2, 64, 16), dtype=np.uint64)
    if lib.kda_trace_read(buf.ctypes.data, buf.size) != buf.size:
        raise SystemExit("kda_trace_read failed")
    print(f"CTA (0, 0), chunks {args.first_chunk} .. {args.first_chunk + 63} "
          f"(SM clock cycles from the chunk's start):")
    _phases(buf[0].astype(np.int64), PREP, "prep warps 0-7")
    _phases(buf[1].astype(np.int64), CHAIN_TRANS, "chain warps 8-15 (transition pass)")


if __name__ == "__main__":
    main()
