"""GPU parity of the fused output gate (kda_fwd_ex / kda_decode out_gate)
against the fp64 oracle, which multiplies its output by the same gate.

Tolerances are the forward pass's (fp32: max |error| <= 1e-4; bf16: relative
Frobenius error per (sequence, head) <= 2e-2).  A gate of ones must leave the
output bit for bit unchanged, and the gate must not touch the state.
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import f32_to_bf16, make_inputs
from kda_testlib import (TOL_BF16_REL_FRO, TOL_F32_MAX_ABS, out_to_f64, rel_fro_per_head,
                         to_device)

pytestmark = pytest.mark.gpu


def _gate(inp, seed, ones=False):
    shape = inp.v.shape
    g = np.ones(shape, np.float32) if ones else \
        np.random.default_rng(seed).uniform(0.0, 1.0, shape).astype(np.float32)
    return f32_to_bf16(g) if inp.bf16 else g


def _dev(a, bf16):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(torch.bfloat16) if bf16 else t).cuda()


def _check(inp, o_g, s_g, gate):
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                inp.cu_seqlens, out_gate=gate)
    o_g = out_to_f64(o_g)
    s_g = s_g.cpu().numpy().astype(np.float64)
    if inp.bf16:
        eo, es = rel_fro_per_head(o_g, o_r, s_g, s_r, inp)
        assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
    else:
        eo = np.abs(o_g.reshape(o_r.shape) - o_r).max()
        es = np.abs(s_g - s_r).max()
        assert eo <= TOL_F32_MAX_ABS and es <= TOL_F32_MAX_ABS, (eo, es)


@pytest.mark.parametrize("seg_chunks", [None, "2"])
def test_gate_tensor_core_path(monkeypatch, seg_chunks):
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    if seg_chunks:
        monkeypatch.setenv("KDA_SEG_CHUNKS", seg_chunks)
    lens = [64 * 5 + 17, 64, 0, 200]
    inp = make_inputs(1, 0, 3, 128, 128, bf16=True, seed=300, seq_lens=lens, state_sigma=0.05,
                      gate_sigma=2.0)
    d = to_device(inp)
    gate = _gate(inp, 1)
    o, s = kda_fwd(**d, out_gate=_dev(gate, True))
    o0, s0 = kda_fwd(**d)
    o1, s1 = kda_fwd(**d, out_gate=_dev(_gate(inp, 0, ones=True), True))
    torch.cuda.synchronize()
    assert torch.equal(o1, o0) and torch.equal(s1, s0) and torch.equal(s, s0)
    _check(inp, o, s, gate)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64)])
def test_gate_cuda_core_path_fp32(dk, dv):
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    inp = make_inputs(2, 64 * 2 + 9, 2, dk, dv, bf16=False, seed=301, state_sigma=0.05)
    d = to_device(inp)
    gate = _gate(inp, 2)
    o, s = kda_fwd(**d, out_gate=_dev(gate, False))
    torch.cuda.synchronize()
    _check(inp, o, s, gate)


@pytest.mark.parametrize("bf16", [True, False])
def test_gate_decode(bf16):
    import torch
    from gated_delta_rule_139_b200 import kda_decode
    inp = make_inputs(6, 5, 2, 128, 128, bf16=bf16, seed=302, state_sigma=0.3)
    d = to_device(inp)
    gate = _gate(inp, 3)
    st = d["initial_state"].clone()
    o, _ = kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st,
                      out_gate=_dev(gate, bf16))
    st0 = d["initial_state"].clone()
    o0, _ = kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st0)
    st1 = d["initial_state"].clone()
    o1, _ = kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st1,
                       out_gate=_dev(_gate(inp, 0, ones=True), bf16))
    torch.cuda.synchronize()
    assert torch.equal(o1, o0) and torch.equal(st, st0) and torch.equal(st1, st0)
    _check(inp, o, st, gate)


def test_gate_with_snapshots():
    """Gate and snapshots together: the snapshots do not see the gate."""
    import torch
    from gated_delta_rule_139_b200 import kda_fwd, kda_fwd_snap
    inp = make_inputs(1, 64 * 6 + 3, 2, 128, 128, bf16=True, seed=303, state_sigma=0.05)
    d = to_device(inp)
    gate = _dev(_gate(inp, 4), True)
    slots = torch.arange(6, dtype=torch.int32, device="cuda").reshape(1, 6)
    pool_g = torch.zeros(6, 2, 128, 128, device="cuda")
    pool = torch.zeros(6, 2, 128, 128, device="cuda")
    o_g, _ = kda_fwd_snap(**d, snap_interval=64, snap_slots=slots, snap_pool=pool_g, out_gate=gate)
    kda_fwd_snap(**d, snap_interval=64, snap_slots=slots, snap_pool=pool)
    o_ref, _ = kda_fwd(**d, out_gate=gate)
    torch.cuda.synchronize()
    assert torch.equal(pool_g, pool) and torch.equal(o_g, o_ref)


def test_fwd_ex_without_options_is_kda_fwd_bitwise():
    import ctypes
    import torch
    import gated_delta_rule_139_b200 as kda
    inp = make_inputs(1, 64 * 3 + 9, 2, 128, 128, bf16=True, seed=304, state_sigma=0.05)
    d = to_device(inp)
    o_ref, s_ref = kda.kda_fwd(**d)
    o = torch.empty_like(o_ref)
    s = torch.empty_like(s_ref)
    dims = kda.Dims(1, inp.T, 2, 128, 128, 0, 1)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = kda.load_library().kda_fwd_ex(P(d["q"]), P(d["k"]), P(d["v"]), P(d["log_alpha"]),
                                       P(d["beta"]), P(d["initial_state"]), None, 64, P(o), P(s),
                                       ctypes.byref(dims), None,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert kda.STATUS[rc] == "KDA_OK"
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


def test_snapshots_and_gate_on_the_cuda_core_path():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd_snap
    inp = make_inputs(2, 64 * 2 + 30, 2, 64, 64, bf16=False, seed=305, state_sigma=0.05)
    d = to_device(inp)
    gate = _gate(inp, 6)
    slots = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    pool = torch.zeros(4, 2, 64, 64, device="cuda")
    o, s = kda_fwd_snap(**d, snap_interval=64, snap_slots=slots, snap_pool=pool,
                        out_gate=_dev(gate, False))
    torch.cuda.synchronize()
    _check(inp, o, s, gate)
    for n in range(2):
        for j in range(2):
            L = 64 * (j + 1)
            sub = lambda a: np.ascontiguousarray(a[n:n + 1, :L])
            _, s_ref = oracle.recurrent(sub(inp.q), sub(inp.k), sub(inp.v), sub(inp.log_alpha),
                                        sub(inp.beta), inp.initial_state[n:n + 1], o_tokens=0)
            assert np.abs(pool[2 * n + j].cpu().numpy() - s_ref[0]).max() <= TOL_F32_MAX_ABS
