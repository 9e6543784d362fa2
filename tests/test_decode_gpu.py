"""GPU parity of the decode / multi-token verify step (kda_decode) against the
fp64 oracle, plus its bookkeeping: in-place state, per-token states, slot table.

A decode step is the recurrence continued from a resident state, so its oracle
is the token-by-token recurrence started from that state.  Tolerances are the
forward pass's: fp32 inputs max |error| <= 1e-4; bf16 inputs relative Frobenius
error <= 2e-2 per (sequence, head) for o and for the updated state.
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, TOL_F32_MAX_ABS, out_to_f64, rel_fro_per_head, to_device

pytestmark = pytest.mark.gpu


def _decode(d, **kw):
    import torch
    from gated_delta_rule_139_b200 import kda_decode
    st = d["initial_state"].clone()
    out, ts = kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], st, **kw)
    torch.cuda.synchronize()
    return out, st, ts


def _compare(inp, o_g, s_g):
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta,
                                inp.initial_state)
    o_g = out_to_f64(o_g)
    s_g = s_g.cpu().numpy().astype(np.float64)
    assert np.isfinite(o_g).all() and np.isfinite(s_g).all()
    if not inp.bf16:
        eo = np.abs(o_g.reshape(o_r.shape) - o_r).max()
        es = np.abs(s_g - s_r).max()
        assert eo <= TOL_F32_MAX_ABS and es <= TOL_F32_MAX_ABS, (eo, es)
    else:
        eo, es = rel_fro_per_head(o_g, o_r, s_g, s_r, inp)
        assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
    return eo, es


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 3, 8, 16])
def test_decode_matches_oracle(bf16, dk, dv, T):
    inp = make_inputs(5, T, 3, dk, dv, bf16=bf16, seed=100 + T + dk + dv, state_sigma=0.3,
                      gate_sigma=2.0)
    o, s, _ = _decode(to_device(inp))
    _compare(inp, o, s)


def test_decode_continues_a_prefill():
    """Prefill 1000 tokens with kda_fwd, then decode 4 more on its final state:
    the outputs and the state match the oracle over all 1004 tokens."""
    import torch
    from gated_delta_rule_139_b200 import kda_fwd
    full = make_inputs(2, 1004, 4, 128, 128, bf16=True, seed=110, state_sigma=0.05)
    d = to_device(full)
    keys = ("q", "k", "v", "log_alpha", "beta")
    pre = {k_: d[k_][:, :1000].contiguous() for k_ in keys}
    dec = {k_: d[k_][:, 1000:].contiguous() for k_ in keys}
    _, state = kda_fwd(**pre, initial_state=d["initial_state"])
    dec["initial_state"] = state
    o, s, _ = _decode(dec)
    o_r, s_r = oracle.recurrent(full.q, full.k, full.v, full.log_alpha, full.beta,
                                full.initial_state)
    o_g = out_to_f64(o)
    for n in range(2):
        for h in range(4):
            ref = o_r[n, 1000:, h]
            assert np.linalg.norm(o_g[n, :, h] - ref) <= TOL_BF16_REL_FRO * np.linalg.norm(ref)
            sr = s_r[n, h]
            sg = s[n, h].cpu().numpy().astype(np.float64)
            assert np.linalg.norm(sg - sr) <= TOL_BF16_REL_FRO * np.linalg.norm(sr)
    torch.cuda.synchronize()


def test_multi_token_equals_single_tokens_bitwise():
    """T tokens in one call give the same bits as T calls of one token."""
    import torch
    from gated_delta_rule_139_b200 import kda_decode
    inp = make_inputs(4, 6, 2, 128, 128, bf16=True, seed=111, state_sigma=0.3)
    d = to_device(inp)
    o_all, s_all, _ = _decode(d)
    st = d["initial_state"].clone()
    outs = []
    for t in range(6):
        sl = lambda x: x[:, t:t + 1].contiguous()
        o, _ = kda_decode(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["log_alpha"]), sl(d["beta"]),
                          st)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, 1), o_all) and torch.equal(st, s_all)


def test_token_states_are_the_prefix_states():
    """token_states[:, t] is the state after tokens 0..t: bitwise equal to a
    call on that prefix, and the last one equals the in-place state."""
    import torch
    inp = make_inputs(3, 5, 2, 128, 64, bf16=True, seed=112, state_sigma=0.3)
    d = to_device(inp)
    o, s, ts = _decode(d, want_token_states=True)
    assert ts.shape == (3, 5, 2, 128, 64)
    assert torch.equal(ts[:, -1], s)
    for t in range(5):
        sub = {k_: d[k_][:, :t + 1].contiguous() for k_ in ("q", "k", "v", "log_alpha", "beta")}
        sub["initial_state"] = d["initial_state"]
        o_t, s_t, _ = _decode(sub)
        assert torch.equal(ts[:, t], s_t) and torch.equal(o[:, :t + 1], o_t)


def test_slot_table_and_padding():
    """Sequences address a state pool through slots; -1 entries touch nothing."""
    import torch
    from gated_delta_rule_139_b200 import kda_decode
    inp = make_inputs(4, 2, 2, 128, 128, bf16=True, seed=113, state_sigma=0.3)
    d = to_device(inp)
    o_ref, s_ref, _ = _decode(d)
    pool = torch.randn(9, 2, 128, 128, device="cuda")
    slot_of = [7, -1, 0, 4]
    for n, sl in enumerate(slot_of):
        if sl >= 0:
            pool[sl] = d["initial_state"][n]
    before = pool.clone()
    slots = torch.tensor(slot_of, dtype=torch.int32, device="cuda")
    out = torch.full_like(o_ref, 7.0)
    kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, slots=slots, out=out)
    torch.cuda.synchronize()
    for n, sl in enumerate(slot_of):
        if sl >= 0:
            assert torch.equal(pool[sl], s_ref[n]) and torch.equal(out[n], o_ref[n])
        else:
            assert (out[n] == 7.0).all()
    for sl in set(range(9)) - {s_ for s_ in slot_of if s_ >= 0}:
        assert torch.equal(pool[sl], before[sl])


def test_out_of_range_slot_sets_the_device_status():
    import torch
    from gated_delta_rule_139_b200 import KDAError, check_device, kda_decode
    inp = make_inputs(2, 1, 1, 128, 128, bf16=True, seed=114, state_sigma=0.3)
    d = to_device(inp)
    check_device()
    pool = d["initial_state"].clone()
    slots = torch.tensor([1, 5], dtype=torch.int32, device="cuda")  # 5 >= pool size 2
    kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, slots=slots)
    with pytest.raises(KDAError) as e:
        check_device()
    assert e.value.name == "KDA_ERR_INVALID_ARG"
    check_device()  # the word was cleared by the read
    assert torch.equal(pool[0], d["initial_state"][0])


def test_decode_gates_are_clamped_bitwise():
    import torch
    inp = make_inputs(2, 4, 2, 128, 128, bf16=True, seed=115, state_sigma=0.3)
    d = to_device(inp)
    rng = np.random.default_rng(1)
    wild = (rng.standard_normal(inp.log_alpha.shape) * 6).astype(np.float32)
    d["log_alpha"] = torch.from_numpy(wild).cuda()
    o1, s1, _ = _decode(d)
    d["log_alpha"] = torch.from_numpy(np.clip(wild, -5, 0)).cuda()
    o2, s2, _ = _decode(d)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_decode_launch_count_and_path():
    from gated_delta_rule_139_b200 import last_launch_count, last_path
    inp = make_inputs(2, 1, 2, 128, 128, bf16=True, seed=116, state_sigma=0.3)
    _decode(to_device(inp))
    assert last_launch_count() == 1 and last_path() == "decode"


def test_decode_fp32_slots_token_states_and_gate_together():
    """Every option at once on the fp32 path: results match the oracle, the
    per-token states are the prefix states, padding entries touch nothing."""
    import torch
    from gated_delta_rule_139_b200 import kda_decode
    inp = make_inputs(3, 5, 2, 64, 128, bf16=False, seed=117, state_sigma=0.3, gate_sigma=2.0)
    d = to_device(inp)
    gate = torch.from_numpy(np.random.default_rng(5).uniform(0, 1, inp.v.shape).astype(np.float32)).cuda()
    pool = torch.zeros(6, 2, 64, 128, device="cuda")
    slot_of = [4, -1, 1]
    for n, sl in enumerate(slot_of):
        if sl >= 0:
            pool[sl] = d["initial_state"][n]
    slots = torch.tensor(slot_of, dtype=torch.int32, device="cuda")
    out = torch.full((3, 5, 2, 128), 9.0, device="cuda")
    _, ts = kda_decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, slots=slots, out=out,
                       out_gate=gate, want_token_states=True)
    torch.cuda.synchronize()
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                out_gate=gate.cpu().numpy())
    for n, sl in enumerate(slot_of):
        if sl < 0:
            assert (out[n] == 9.0).all()
            continue
        assert np.abs(out[n].cpu().numpy() - o_r[n]).max() <= TOL_F32_MAX_ABS
        assert np.abs(pool[sl].cpu().numpy() - s_r[n]).max() <= TOL_F32_MAX_ABS
        assert torch.equal(ts[n, -1], pool[sl])
        for t in range(5):
            sub = lambda a: np.ascontiguousarray(a[n:n + 1, :t + 1])
            _, s_t = oracle.recurrent(sub(inp.q), sub(inp.k), sub(inp.v), sub(inp.log_alpha),
                                      sub(inp.beta), inp.initial_state[n:n + 1], o_tokens=0)
            assert np.abs(ts[n, t].cpu().numpy() - s_t[0]).max() <= TOL_F32_MAX_ABS
