"""A seeded synthetic kda_fwd case of chosen size, for profilers.

    python -m gated_delta_rule_139_b200.profile_case [--B 1] [--T 16384] [--H 32] [--calls 2]

Builds bf16 q/k/v (d_k = d_v = 128) and fp32 gates with the distributions of the
long-prefill workload, uploads them, and runs kda_fwd `--calls` times on cuda:0
with a synchronize after each call, so that a profiler can skip the first call's
launches and capture a later one.  Prints the launches of the last call.
"""
from __future__ import annotations

import argparse

import numpy as np


def main(argv=None) -> None:
    import torch

    import gated_delta_rule_139_b200 as kda
    from gated_delta_rule_139_b200.inputs import make_inputs

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--calls", type=int, default=2)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)
    inp = make_inputs(args.B, args.T, args.H, 128, 128, bf16=True, seed=args.seed, gate_mu=-1.0,
                      gate_sigma=1.0)
    dev = torch.device("cuda", 0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q, k, v = t(inp.q), t(inp.k), t(inp.v)
    la, be = f(inp.log_alpha), f(inp.beta)
    for _ in range(args.calls):
        kda.kda_fwd(q, k, v, la, be)
        torch.cuda.synchronize(dev)
    kda.check_device()
    print(f"profile_case B={args.B} T={args.T} H={args.H}: {args.calls} calls, "
          f"{kda.last_launch_count()} launches each, path {kda.last_path()}")


if __name__ == "__main__":
    main()
