"""Context-parallel prefill on CPU ranks (gloo): the orchestration of
gated_delta_rule_139_b200.cp -- span transitions, one all-gather, the prefix
scan over earlier ranks, the forward pass from the recovered state -- with the
three per-rank steps done by the fp64 oracle.

The transition of a span is measured from the oracle itself (B = final state
from a zero state; column i of M from a unit state), so this checks the affine
decomposition of the recurrence (the chunk-parallel section of the aiblin.ru
page) as well as the collective pattern: the concatenated span outputs and the
last rank's state must equal the oracle run over the whole sequences.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

B, H, DK, DV, SPAN = 2, 2, 8, 6, 37


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world):
    from gated_delta_rule_139_b200.inputs import make_inputs
    return make_inputs(B, SPAN * world, H, DK, DV, bf16=False, seed=500 + world,
                       state_sigma=0.3, gate_sigma=1.5)


def _oracle_ops():
    import oracle
    from gated_delta_rule_139_b200.cp import SpanOps

    npy = lambda t: t.numpy()

    def transition(q, k, v, la, be):
        kw = dict(q=npy(k), k=npy(k), v=npy(v), log_alpha=npy(la), beta=npy(be), o_tokens=0)
        _, b = oracle.recurrent(initial_state=None, **kw)
        m = np.empty((B, H, DK, DK))
        for i in range(DK):  # S_out(E_i0) - B = M E_i0: column i of M in column 0
            e = np.zeros((B, H, DK, DV), np.float32)
            e[:, :, i, 0] = 1.0
            _, s = oracle.recurrent(initial_state=e, **kw)
            m[:, :, :, i] = s[:, :, :, 0] - b[:, :, :, 0]
        return torch.from_numpy(np.concatenate([m, b], axis=3)), None  # [B,H,dk,dk+dv] = [M | B]

    def apply(prior, s0):
        s = np.zeros((B, H, DK, DV)) if s0 is None else s0.numpy().astype(np.float64)
        for j in range(prior.shape[0]):
            m, b = prior[j, ..., :DK].numpy(), prior[j, ..., DK:].numpy()
            s = np.einsum("bhij,bhjv->bhiv", m, s) + b
        return s

    def forward(q, k, v, la, be, s_in, gate, ctx):
        o, s = oracle.recurrent(npy(q), npy(k), npy(v), npy(la), npy(be),
                                s_in.astype(np.float32), o_tokens=None,
                                out_gate=None if gate is None else npy(gate))
        return torch.from_numpy(o), torch.from_numpy(s)

    return SpanOps(transition, apply, forward)


def _gate(world):
    return np.random.default_rng(600 + world).uniform(0, 1, (B, SPAN * world, H, DV)).astype(np.float32)


def _rank(rank, world, port, q, gated=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from gated_delta_rule_139_b200.cp import cp_prefill
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _inputs(world)
        sl = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, rank * SPAN:(rank + 1) * SPAN]))
        o, s = cp_prefill(sl(x.q), sl(x.k), sl(x.v), sl(x.log_alpha), sl(x.beta),
                          torch.from_numpy(x.initial_state), ops=_oracle_ops(),
                          out_gate=sl(_gate(world)) if gated else None)
        q.put((rank, o.numpy(), s.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,gated", [(2, False), (3, False), (4, False), (2, True)])
def test_cp_prefill_on_gloo_ranks_matches_the_whole_sequence(world, gated):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, gated)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, o, s = q.get(timeout=180)
        got[rank] = (o, s)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x = _inputs(world)
    o_ref, s_ref = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.beta, x.initial_state,
                                    out_gate=_gate(world) if gated else None)
    o_cp = np.concatenate([got[r][0] for r in range(world)], axis=1)
    # the oracle takes its initial state in fp32, so the recovered state enters each
    # span rounded to fp32 (relative 2^-24); a structural mistake would be O(1)
    tol = 1e-6
    assert np.abs(o_cp - o_ref).max() <= tol * np.abs(o_ref).max()
    assert np.abs(got[world - 1][1] - s_ref).max() <= tol * np.abs(s_ref).max()
    # every other rank ends at the state entering the next span
    for r in range(world - 1):
        _, s_mid = oracle.recurrent(x.q[:, :SPAN * (r + 1)], x.k[:, :SPAN * (r + 1)],
                                    x.v[:, :SPAN * (r + 1)], x.log_alpha[:, :SPAN * (r + 1)],
                                    x.beta[:, :SPAN * (r + 1)], x.initial_state)
        assert np.abs(got[r][1] - s_mid).max() <= tol * np.abs(s_mid).max()
