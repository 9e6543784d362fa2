"""GPU parity: libkda.so (through the C ABI) against the fp64 oracle.

Tolerances: fp32 inputs max |error| <= 1e-4 on every output and final-state
element; bf16 inputs relative Frobenius error <= 2e-2 per (sequence, head) for o
(over tokens x d_v) and for the final state, and <= 4e-2 per 64-token chunk of
each (sequence, head) (denominator floored at a quarter of the head's RMS).
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs, workload
from kda_testlib import (TOL_BF16_REL_FRO, TOL_BF16_REL_FRO_CHUNK, TOL_F32_MAX_ABS,
                         rel_fro_per_chunk, rel_fro_per_head, run_gpu, to_device, out_to_f64)

pytestmark = pytest.mark.gpu


def _oracle(inp, o_tokens=None):
    return oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                            inp.cu_seqlens, o_tokens=o_tokens)


def _check(inp, o_tokens=None, tol=None):
    o_g, s_g = run_gpu(inp)
    o_r, s_r = _oracle(inp, o_tokens)
    if o_tokens is not None:
        o_g = o_g.reshape(-1, inp.H, inp.dv)[:o_tokens]
    assert np.isfinite(o_g).all() and np.isfinite(s_g).all()
    if not inp.bf16:
        err_o = np.abs(o_g.reshape(o_r.shape) - o_r).max()
        err_s = np.abs(s_g - s_r).max()
        assert err_o <= (tol or TOL_F32_MAX_ABS), err_o
        assert err_s <= (tol or TOL_F32_MAX_ABS), err_s
        return err_o, err_s
    eo, es = rel_fro_per_head(o_g, o_r, s_g, s_r, inp, o_tokens)
    ec, where = rel_fro_per_chunk(o_g, o_r, inp, o_tokens)
    assert eo <= (tol or TOL_BF16_REL_FRO), eo
    assert es <= (tol or TOL_BF16_REL_FRO), es
    assert ec <= TOL_BF16_REL_FRO_CHUNK, (ec, "(sequence, chunk, head)", where)
    return eo, es, ec


# ---------------------------------------------------------------- the five workloads
def test_workload_tiny_fp32():
    print(_check(workload("tiny_fp32")))


def test_workload_b2_t4k():
    print(_check(workload("b2_t4k")))


def test_workload_prefill_64k():
    print(_check(workload("prefill_64k")))


def test_workload_packed_16():
    print(_check(workload("packed_16")))


def test_workload_prefill_1m_first_64k_and_final_state():
    print(_check(workload("prefill_1m"), o_tokens=65536))


# ---------------------------------------------------------------- small cases, edges
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_ragged_tails(bf16, dk, dv):
    # T not a multiple of the chunk; several chunks; two batch entries
    inp = make_inputs(2, 64 * 3 + 17, 3, dk, dv, bf16=bf16, seed=dk + dv, state_sigma=0.05,
                      gate_sigma=2.0)
    _check(inp)


@pytest.mark.parametrize("bf16", [False, True])
def test_packed_with_empty_and_tiny_sequences(bf16):
    lens = [0, 1, 63, 64, 65, 0, 200, 7]
    inp = make_inputs(1, 0, 4, 128, 128, bf16=bf16, seed=21, seq_lens=lens, state_sigma=0.05)
    o_g, s_g = run_gpu(inp)
    _check(inp)
    # a zero-length sequence returns its initial state unchanged
    np.testing.assert_array_equal(s_g[0], inp.initial_state[0].astype(np.float64))
    np.testing.assert_array_equal(s_g[5], inp.initial_state[5].astype(np.float64))


def test_clamp_floor_and_one_everywhere():
    inp = make_inputs(1, 64 * 4 + 5, 2, 128, 128, bf16=True, seed=22, state_sigma=0.05)
    la = inp.log_alpha
    la[..., ::2] = -5.0
    la[..., 1::2] = 0.0
    _check(inp)


def test_out_of_range_gates_equal_their_clamp_bitwise():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    inp = make_inputs(1, 300, 2, 128, 128, bf16=True, seed=23, state_sigma=0.05)
    rng = np.random.default_rng(0)
    wild = (rng.standard_normal(inp.log_alpha.shape) * 6).astype(np.float32)
    d = to_device(inp)
    d["log_alpha"] = torch.from_numpy(wild).cuda()
    o1, s1 = kda_fwd(**d)
    d["log_alpha"] = torch.from_numpy(np.clip(wild, -5, 0)).cuda()
    o2, s2 = kda_fwd(**d)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_deterministic_bitwise():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    inp = make_inputs(1, 1000, 4, 128, 128, bf16=True, seed=24, state_sigma=0.05)
    d = to_device(inp)
    o1, s1 = kda_fwd(**d)
    o2, s2 = kda_fwd(**d)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_packed_equals_separate_bitwise():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    lens = [130, 64, 257]
    inp = make_inputs(1, 0, 2, 128, 128, bf16=True, seed=25, seq_lens=lens, state_sigma=0.05)
    d = to_device(inp)
    o, s = kda_fwd(**d)
    cu = inp.cu_seqlens
    for n in range(len(lens)):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        on, sn = kda_fwd(d["q"][None, sl].contiguous(), d["k"][None, sl].contiguous(),
                         d["v"][None, sl].contiguous(), d["log_alpha"][None, sl].contiguous(),
                         d["beta"][None, sl].contiguous(), d["initial_state"][n:n + 1].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(on[0], o[sl]) and torch.equal(sn[0], s[n])


def test_resume_from_final_state(monkeypatch):
    """Split at a chunk boundary with final -> initial state: identical to one call
    when neither call is cut into segments (same chunks, same arithmetic)."""
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    monkeypatch.setenv("KDA_SEG_CHUNKS", "100000")
    inp = make_inputs(1, 640, 2, 128, 128, bf16=True, seed=26, state_sigma=0.05)
    d = to_device(inp)
    o, s = kda_fwd(**d)
    T1 = 320
    keys = ("q", "k", "v", "log_alpha", "beta")
    a = {k_: d[k_][:, :T1].contiguous() for k_ in keys}
    b = {k_: d[k_][:, T1:].contiguous() for k_ in keys}
    o1, s1 = kda_fwd(**a, initial_state=d["initial_state"])
    o2, s2 = kda_fwd(**b, initial_state=s1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], 1), o) and torch.equal(s2, s)


@pytest.mark.parametrize("seg_chunks", ["1", "2", "3", "5"])
def test_segment_split_matches_oracle(monkeypatch, seg_chunks):
    """Forced segment lengths: the segment transitions (local state + transition
    matrix) and their scan reassemble the sequential result."""
    monkeypatch.setenv("KDA_SEG_CHUNKS", seg_chunks)
    lens = [64 * 7 + 5, 64, 0, 64 * 3, 31]
    inp = make_inputs(1, 0, 3, 128, 128, bf16=True, seed=31, seq_lens=lens, state_sigma=0.05,
                      gate_sigma=2.0)
    _check(inp)
    inp2 = make_inputs(2, 64 * 6 + 9, 2, 128, 128, bf16=True, seed=32, state_sigma=0.05)
    _check(inp2)


def test_segment_split_in_place_state(monkeypatch):
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    monkeypatch.setenv("KDA_SEG_CHUNKS", "2")
    inp = make_inputs(1, 64 * 9, 2, 128, 128, bf16=True, seed=33, state_sigma=0.05)
    d = to_device(inp)
    o, s = kda_fwd(**d)
    st = d["initial_state"].clone()
    o2, _ = kda_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(s, st)


def test_device_status_clean():
    from gated_delta_rule_139_b200 import check_device
    inp = make_inputs(1, 300, 2, 128, 128, bf16=True, seed=34)
    run_gpu(inp)
    check_device()


def test_state_in_place():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    inp = make_inputs(1, 200, 2, 128, 128, bf16=True, seed=27, state_sigma=0.05)
    d = to_device(inp)
    o, s = kda_fwd(**d)
    st = d["initial_state"].clone()
    o2, s2 = kda_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert s2.data_ptr() == st.data_ptr()
    assert torch.equal(o, o2) and torch.equal(s, st)


def test_no_final_state_requested():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    inp = make_inputs(1, 130, 2, 128, 128, bf16=True, seed=28)
    d = to_device(inp)
    o, _ = kda_fwd(**d)
    o2, s2 = kda_fwd(**d, want_final=False)
    torch.cuda.synchronize()
    assert s2 is None and torch.equal(o, o2)


def test_host_entry_point_matches_device_entry_point():
    import torch
    from gated_delta_rule_139_b200 import kda_fwd, kda_fwd_host
    inp = make_inputs(1, 0, 2, 128, 128, bf16=True, seed=29, seq_lens=[100, 300],
                      state_sigma=0.05)
    o_h, s_h = kda_fwd_host(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                            inp.cu_seqlens)
    d = to_device(inp)
    o_d, s_d = kda_fwd(**d)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(o_h, o_d.view(torch.int16).cpu().numpy().view(np.uint16))
    np.testing.assert_array_equal(s_h, s_d.cpu().numpy())


def test_host_pointer_is_rejected():
    import ctypes
    import gated_delta_rule_139_b200 as kda
    inp = make_inputs(1, 64, 1, 128, 128, bf16=True, seed=30)
    out = np.empty_like(inp.v)
    d = kda.Dims(1, 64, 1, 128, 128, 0, 1)
    P = lambda a: ctypes.c_void_p(a.ctypes.data)
    rc = kda.load_library().kda_fwd(P(inp.q), P(inp.k), P(inp.v), P(inp.log_alpha), P(inp.beta),
                                    None, None, 64, P(out), None, ctypes.byref(d), None)
    assert kda.STATUS[rc] == "KDA_ERR_INVALID_ARG"


@pytest.mark.parametrize("bf16,d", [(True, 128), (False, 64)])
def test_host_entry_point_pipelines_long_sequences_in_spans(monkeypatch, bf16, d):
    """One long sequence through kda_fwd_host runs as spans (here 512 tokens): the
    result is bit for bit kda_fwd called span after span with the state carried,
    and matches the oracle over the whole sequence."""
    import torch
    from gated_delta_rule_139_b200 import kda_fwd, kda_fwd_host, last_launch_count
    monkeypatch.setenv("KDA_HOST_SPAN_TOKENS", "512")
    T = 64 * 37 + 21  # four full spans and a ragged fifth
    inp = make_inputs(1, T, 2, d, d, bf16=bf16, seed=31, state_sigma=0.05, gate_sigma=2.0)
    o_h, s_h = kda_fwd_host(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)
    assert last_launch_count() >= 5
    dd = to_device(inp)
    state = dd["initial_state"]
    outs = []
    for t0 in range(0, T, 512):
        sl = {k_: dd[k_][:, t0:t0 + 512].contiguous() for k_ in ("q", "k", "v", "log_alpha", "beta")}
        o, state = kda_fwd(**sl, initial_state=state)
        outs.append(o)
    torch.cuda.synchronize()
    o_d = torch.cat(outs, 1)
    o_d = o_d.view(torch.int16).cpu().numpy().view(np.uint16) if bf16 else o_d.cpu().numpy()
    np.testing.assert_array_equal(o_h, o_d)
    np.testing.assert_array_equal(s_h, state.cpu().numpy())
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)
    og = out_to_f64(torch.from_numpy(o_h.view(np.int16)).view(torch.bfloat16) if bf16
                    else torch.from_numpy(o_h))
    if bf16:
        eo, es = rel_fro_per_head(og, o_r, s_h.astype(np.float64), s_r, inp)
        assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
    else:
        assert np.abs(og.reshape(o_r.shape) - o_r).max() <= TOL_F32_MAX_ABS
        assert np.abs(s_h - s_r).max() <= TOL_F32_MAX_ABS


def test_packed_one_long_and_many_short_sequences(monkeypatch):
    """One long sequence cut into segments beside 300 short ones: the chunk cache is
    indexed by each segment's first chunk among all chunks (the short sequences' units
    take one entry each), and every output and final state matches the oracle."""
    monkeypatch.setenv("KDA_SEG_CHUNKS", "4")
    lens = [64 * 40 + 7] + [1 + (37 * i) % 150 for i in range(300)]
    inp = make_inputs(1, 0, 2, 128, 128, bf16=True, seed=33, seq_lens=lens, state_sigma=0.05,
                      gate_sigma=2.0)
    _check(inp)
