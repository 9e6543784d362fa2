"""GPU parity of the context-parallel pieces: span transitions
(kda_transition), chains of them (kda_apply_transitions), and the whole
context-parallel prefill emulated on one GPU -- the virtual ranks run one after
another, the all-gather is a stack of their transitions -- against the fp64
oracle.  The real collective path runs with a one-rank NCCL group.

Tolerance: relative Frobenius error per (sequence, head) <= 2e-2 (bf16 inputs).
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, out_to_f64, to_device

pytestmark = pytest.mark.gpu


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _worst_state_err(got, ref):
    return max(_rel(got[n, h], ref[n, h]) for n in range(ref.shape[0]) for h in range(ref.shape[1]))


@pytest.mark.parametrize("seg_chunks", [None, "2", "3"])
def test_transition_is_the_spans_affine_map(monkeypatch, seg_chunks):
    """B = the state reached from zero; M S + B = the state reached from S."""
    import torch
    from gated_delta_rule_139_b200 import kda_apply_transitions, kda_transition
    if seg_chunks:
        monkeypatch.setenv("KDA_SEG_CHUNKS", seg_chunks)
    inp = make_inputs(2, 64 * 9 + 13, 2, 128, 128, bf16=True, seed=400, state_sigma=0.1,
                      gate_sigma=2.0)
    d = to_device(inp)
    trans = kda_transition(d["k"], d["v"], d["log_alpha"], d["beta"])
    from_zero = kda_apply_transitions(trans[None])
    from_s = kda_apply_transitions(trans[None], d["initial_state"])
    torch.cuda.synchronize()
    _, b_ref = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, o_tokens=0)
    _, s_ref = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                o_tokens=0)
    bt = trans[:, :, 0].transpose(-1, -2).cpu().numpy().astype(np.float64)
    assert _worst_state_err(bt, b_ref) <= TOL_BF16_REL_FRO
    assert _worst_state_err(from_zero.cpu().numpy().astype(np.float64), b_ref) <= TOL_BF16_REL_FRO
    assert _worst_state_err(from_s.cpu().numpy().astype(np.float64), s_ref) <= TOL_BF16_REL_FRO


def test_empty_span_is_the_identity_map():
    import torch
    from gated_delta_rule_139_b200 import kda_apply_transitions, kda_transition
    inp = make_inputs(1, 0, 2, 128, 128, bf16=True, seed=401, state_sigma=0.1)
    d = to_device(inp)
    e = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    trans = kda_transition(e, e, torch.empty(1, 0, 2, 128, device="cuda"),
                           torch.empty(1, 0, 2, device="cuda"))
    out = kda_apply_transitions(trans[None], d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(trans[:, :, 0], torch.zeros_like(trans[:, :, 0]))
    assert torch.equal(trans[:, :, 1], torch.eye(128, device="cuda").expand_as(trans[:, :, 1]))
    assert torch.equal(out, d["initial_state"])


def test_apply_zero_transitions_copies_and_works_in_place():
    import torch
    from gated_delta_rule_139_b200 import kda_apply_transitions, kda_transition
    inp = make_inputs(2, 300, 2, 128, 128, bf16=True, seed=402, state_sigma=0.1)
    d = to_device(inp)
    s0 = d["initial_state"]
    none = torch.empty(0, 2, 2, 2, 128, 128, device="cuda")
    assert torch.equal(kda_apply_transitions(none, s0), s0)
    assert torch.equal(kda_apply_transitions(none), torch.zeros_like(s0))
    trans = kda_transition(d["k"], d["v"], d["log_alpha"], d["beta"])
    ref = kda_apply_transitions(trans[None], s0)
    st = s0.clone()
    kda_apply_transitions(trans[None], st, out=st)
    torch.cuda.synchronize()
    assert torch.equal(st, ref)


@pytest.mark.parametrize("world", [2, 4])
def test_context_parallel_prefill_emulated_on_one_gpu(world):
    """Virtual ranks one after another on one GPU: their concatenated outputs
    and the last rank's state match the oracle over the whole sequences."""
    import torch
    from gated_delta_rule_139_b200 import (kda_apply_transitions, kda_span_forward,
                                           kda_span_transition, span_workspace)
    span = 64 * 5 + 7
    inp = make_inputs(2, span * world, 2, 128, 128, bf16=True, seed=403 + world,
                      state_sigma=0.05, gate_sigma=2.0)
    d = to_device(inp)
    keys = ("q", "k", "v", "log_alpha", "beta")
    spans = [{k_: d[k_][:, r * span:(r + 1) * span].contiguous() for k_ in keys}
             for r in range(world)]
    ws = [span_workspace(s["k"]) for s in spans]
    trans = [kda_span_transition(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], w)
             for s, w in zip(spans, ws)]
    gathered = torch.stack(trans)  # what the all-gather delivers
    outs, finals = [], []
    for r, s in enumerate(spans):
        s_in = kda_apply_transitions(gathered[:r], d["initial_state"])
        o, f = kda_span_forward(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], ws[r], s_in)
        outs.append(o)
        finals.append(f)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                    inp.initial_state)
    o_cp = out_to_f64(torch.cat(outs, 1))
    for n in range(2):
        for h in range(2):
            assert _rel(o_cp[n, :, h], o_ref[n, :, h]) <= TOL_BF16_REL_FRO
    assert _worst_state_err(finals[-1].cpu().numpy().astype(np.float64), s_ref) <= TOL_BF16_REL_FRO


@pytest.mark.parametrize("seg_chunks", [None, "2"])
def test_span_transition_and_forward_share_the_work(monkeypatch, seg_chunks):
    """kda_span_transition fills the workspace; kda_span_forward from it gives
    kda_fwd's results (bit for bit when the span is cut into segments, where
    kda_fwd runs the same scan and forward pass; within tolerance otherwise) and
    the transition equals kda_transition's."""
    import torch
    from gated_delta_rule_139_b200 import (kda_fwd, kda_span_forward, kda_span_transition,
                                           kda_transition, span_workspace)
    if seg_chunks:
        monkeypatch.setenv("KDA_SEG_CHUNKS", seg_chunks)
    inp = make_inputs(2, 64 * 7 + 11, 2, 128, 128, bf16=True, seed=420, state_sigma=0.05,
                      gate_sigma=2.0)
    d = to_device(inp)
    keys = ("q", "k", "v", "log_alpha", "beta")
    ws = span_workspace(d["k"])
    trans = kda_span_transition(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws)
    trans_ref = kda_transition(d["k"], d["v"], d["log_alpha"], d["beta"])
    o, f = kda_span_forward(*(d[k_] for k_ in keys), ws, d["initial_state"])
    o2, f2 = kda_span_forward(*(d[k_] for k_ in keys), ws, d["initial_state"])  # reusable
    o_ref, f_ref = kda_fwd(**{k_: d[k_] for k_ in keys}, initial_state=d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(trans, trans_ref)
    assert torch.equal(o, o2) and torch.equal(f, f2)
    if seg_chunks:
        assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
    o_or, s_or = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)
    o_g = out_to_f64(o)
    for n in range(2):
        for h in range(2):
            assert _rel(o_g[n, :, h], o_or[n, :, h]) <= TOL_BF16_REL_FRO
    assert _worst_state_err(f.cpu().numpy().astype(np.float64), s_or) <= TOL_BF16_REL_FRO


def test_cp_prefill_through_a_one_rank_nccl_group(monkeypatch):
    """The collective code path with real kernels: one rank, with the span cut
    into segments (so kda_fwd takes the same segmented path), so it must equal
    kda_fwd bit for bit."""
    import torch
    import torch.distributed as dist
    from gated_delta_rule_139_b200 import kda_fwd
    from gated_delta_rule_139_b200.cp import cp_prefill
    monkeypatch.setenv("KDA_SEG_CHUNKS", "2")
    inp = make_inputs(1, 64 * 4 + 5, 2, 128, 128, bf16=True, seed=410, state_sigma=0.05)
    d = to_device(inp)
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        o, f = cp_prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["initial_state"])
        o_ref, f_ref = kda_fwd(**{k_: d[k_] for k_ in ("q", "k", "v", "log_alpha", "beta")},
                               initial_state=d["initial_state"])
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
    finally:
        dist.destroy_process_group()


def test_cp_prefill_with_output_gate(monkeypatch):
    """The gated forward through the collective path: one rank, segmented span,
    so it must equal kda_fwd with the same gate bit for bit."""
    import torch
    import torch.distributed as dist
    from gated_delta_rule_139_b200 import kda_fwd
    from gated_delta_rule_139_b200.cp import cp_prefill
    monkeypatch.setenv("KDA_SEG_CHUNKS", "2")
    inp = make_inputs(1, 64 * 5 + 3, 2, 128, 128, bf16=True, seed=411, state_sigma=0.05)
    d = to_device(inp)
    gate = torch.rand(inp.v.shape, device="cuda").to(torch.bfloat16)
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        keys = ("q", "k", "v", "log_alpha", "beta")
        o, f = cp_prefill(*(d[k_] for k_ in keys), d["initial_state"], out_gate=gate)
        o_ref, f_ref = kda_fwd(**{k_: d[k_] for k_ in keys}, initial_state=d["initial_state"],
                               out_gate=gate)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
    finally:
        dist.destroy_process_group()


def test_span_forward_with_gate_and_snapshots_equals_kda_fwd(monkeypatch):
    """kda_span_forward_ex from the workspace: with the span cut into segments it
    takes kda_fwd's segmented path, so output, state and snapshots equal
    kda_fwd_snap's with the same gate bit for bit."""
    import torch
    from gated_delta_rule_139_b200 import (kda_fwd_snap, kda_span_forward, kda_span_transition,
                                           span_workspace)
    monkeypatch.setenv("KDA_SEG_CHUNKS", "2")
    inp = make_inputs(2, 64 * 7 + 11, 2, 128, 128, bf16=True, seed=421, state_sigma=0.05,
                      gate_sigma=2.0)
    d = to_device(inp)
    keys = ("q", "k", "v", "log_alpha", "beta")
    gate = torch.rand(inp.v.shape, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([[0, -1, 1], [2, 3, 4]], dtype=torch.int32, device="cuda")
    pools = [torch.full((6, 2, 128, 128), 3.0, device="cuda") for _ in range(2)]
    ws = span_workspace(d["k"])
    kda_span_transition(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws)
    o, f = kda_span_forward(*(d[k_] for k_ in keys), ws, d["initial_state"], out_gate=gate,
                            snap_interval=128, snap_slots=slots, snap_pool=pools[0])
    o_ref, f_ref = kda_fwd_snap(**{k_: d[k_] for k_ in keys}, initial_state=d["initial_state"],
                                snap_interval=128, snap_slots=slots, snap_pool=pools[1],
                                out_gate=gate)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
    assert torch.equal(pools[0], pools[1])
    assert (pools[0][5] == 3.0).all()  # unused slot untouched


def test_cp_snapshots_at_span_aligned_positions(monkeypatch):
    """Two virtual ranks whose spans start at multiples of the interval: each
    rank's snapshots (positions counted from its span's start) are the oracle's
    prefix states at the matching whole-sequence positions."""
    import torch
    from gated_delta_rule_139_b200 import (kda_apply_transitions, kda_span_forward,
                                           kda_span_transition, span_workspace)
    monkeypatch.setenv("KDA_SEG_CHUNKS", "2")
    span, interval = 64 * 4, 128
    inp = make_inputs(1, 2 * span, 2, 128, 128, bf16=True, seed=422, state_sigma=0.05,
                      gate_sigma=2.0)
    d = to_device(inp)
    keys = ("q", "k", "v", "log_alpha", "beta")
    spans = [{k_: d[k_][:, r * span:(r + 1) * span].contiguous() for k_ in keys} for r in range(2)]
    ws = [span_workspace(s["k"]) for s in spans]
    trans = torch.stack([kda_span_transition(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"], w)
                         for s, w in zip(spans, ws)])
    pool = torch.zeros(4, 2, 128, 128, device="cuda")
    for r, s in enumerate(spans):
        s_in = kda_apply_transitions(trans[:r], d["initial_state"])
        sl = torch.tensor([[2 * r, 2 * r + 1]], dtype=torch.int32, device="cuda")
        kda_span_forward(*(s[k_] for k_ in keys), ws[r], s_in, snap_interval=interval,
                         snap_slots=sl, snap_pool=pool)
    torch.cuda.synchronize()
    got = pool.cpu().numpy().astype(np.float64)
    for j in range(4):  # whole-sequence positions 128, 256, 384, 512
        L = (j + 1) * interval
        _, ref = oracle.recurrent(inp.q[:, :L], inp.k[:, :L], inp.v[:, :L], inp.log_alpha[:, :L],
                                  inp.beta[:, :L], inp.initial_state, o_tokens=0)
        for h in range(2):
            assert _rel(got[j, h], ref[0, h]) <= TOL_BF16_REL_FRO, (j, h)


# ---------------------------------------------------------------- the chunkwise operands
# kda_chunk_operands writes, per chunk and head, one 74 240-byte entry of bf16 operand images
# as they sit in shared memory, with the 128-byte swizzle of the tensor-core operand layouts:
#   K-major (rows r, K index k):  (k // 64) R 128 + (r // 8) 1024 + (r % 8) 128
#                                 + (((k % 64) // 8) ^ (r % 8)) 16 + (k % 8) 2
#   MN-major (K rows k, MN index m): the same with (r, k) -> (k, m) and R -> K rows
# at offsets W^T 0 (MN-major, K rows = channels), U'^T 16K ([128][64], 16-byte pieces of
# row e XOR-swizzled by e % 8), K_dec 32K (MN-major, K rows = tokens), Q~ 48K (K-major),
# P 64K (K-major 64 x 64), gamma 72K (fp32 [128]).
_CI = {"W": 0, "U": 16384, "Kdec": 32768, "Qt": 49152, "P": 65536, "gamma": 73728}
_ENTRY = 74240


def _swz(r, k, R):
    return (k // 64) * R * 128 + (r // 8) * 1024 + (r % 8) * 128 + (((k % 64) // 8) ^ (r % 8)) * 16 + \
        (k % 8) * 2


def _offsets():
    """Byte offsets of each piece's elements, as [rows, cols] of the operand (tokens first)."""
    t = np.arange(64)[:, None]
    c = np.arange(128)[None, :]
    s = np.arange(64)[None, :]
    return {"W": _CI["W"] + _swz(c, t, 128),               # W[t][c] = W^T[c][t], MN-major
            "U": _CI["U"] + c * 128 + (((t // 8) ^ (c % 8)) << 4) + (t % 8) * 2,  # U'[t][e]
            "Kdec": _CI["Kdec"] + _swz(t, c, 64),          # K_dec[t][c], MN-major (K rows = t)
            "Qt": _CI["Qt"] + _swz(t, c, 64),              # Q~[t][c], K-major
            "P": _CI["P"] + _swz(t, s, 64)}                # P[t][s], K-major


def _decode_entry(entry):
    """{name: float32 array} of one entry (uint8 [74240])."""
    out = {}
    for name, off in _offsets().items():
        lo, hi = entry[off].astype(np.uint32), entry[off + 1].astype(np.uint32)
        out[name] = ((hi << 24) | (lo << 16)).view(np.float32)
    out["gamma"] = entry[_CI["gamma"]:_CI["gamma"] + 512].view(np.float32).copy()
    return out


@pytest.mark.parametrize("gate_sigma,pin", [(2.0, None), (1.0, "floor"), (1.0, "mixed")])
def test_chunk_operands_match_the_oracle(gate_sigma, pin):
    """kda_chunk_operands gives every chunk's W, U', K_dec, Q~, P and gamma as the forward
    pass hands them to its state products; decoded from their operand images they match the
    fp64 chunkwise operands of the oracle (two sequences of 3 full chunks and a ragged one,
    two heads; bf16 operands: relative Frobenius error per chunk and head <= 2e-2; gamma
    within 1e-4).  pin="floor": every gate at the clamp floor (the in-chunk decay reaches
    e^-315); pin="mixed": half the channels at the floor, half at log alpha = 0."""
    import torch
    from gated_delta_rule_139_b200 import kda_chunk_operands
    T, H, B = 64 * 3 + 5, 2, 2
    inp = make_inputs(B, T, H, 128, 128, bf16=True, seed=430, gate_sigma=gate_sigma)
    if pin == "floor":
        inp.log_alpha[...] = -5.0
    elif pin == "mixed":
        inp.log_alpha[..., 0::2] = -5.0
        inp.log_alpha[..., 1::2] = 0.0
    d = to_device(inp)
    raw = kda_chunk_operands(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"]).cpu().numpy()
    torch.cuda.synchronize()
    nch = 4
    assert raw.shape == (B * nch * H, _ENTRY)
    for b in range(B):
        ref = oracle.chunk_operands(inp.q[b:b + 1], inp.k[b:b + 1], inp.v[b:b + 1],
                                    inp.log_alpha[b:b + 1], inp.beta[b:b + 1], 64)
        for c in range(nch):
            for h in range(H):
                got = _decode_entry(raw[(b * nch + c) * H + h])
                for name in ("W", "U", "Kdec", "Qt", "P"):
                    g, r = got[name].astype(np.float64), ref[name][c, h]
                    assert np.isfinite(g).all(), (b, c, h, name)
                    assert _rel(g, r) <= TOL_BF16_REL_FRO, (b, c, h, name, _rel(g, r))
                # gamma = e^{g_last} in fp32 (the sum of up to 64 fp32 gates; strong decay may
                # fall below fp32's normal range and flush to zero, which is the right limit)
                np.testing.assert_allclose(got["gamma"], ref["gamma"][c, h], rtol=1e-4, atol=1e-6)
