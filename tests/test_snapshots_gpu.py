"""GPU parity of the prefix-cache state snapshots (kda_fwd_snap).

Snapshot j of sequence n is the state after its first (j+1)*interval tokens;
its oracle is the fp64 token recurrence run on that prefix.  Tolerances are the
forward pass's (fp32: max |error| <= 1e-4; bf16: relative Frobenius error per
head <= 2e-2).
"""
import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, TOL_F32_MAX_ABS, seq_bounds, to_device

pytestmark = pytest.mark.gpu


def _prefix_state(inp, n, L):
    """Oracle state of sequence n after its first L tokens."""
    lo, _ = seq_bounds(inp)[n]  # first token of the sequence in the flattened token axis
    H = inp.H

    def sl(a, per_token):  # tokens lo .. lo+L-1 of a token-major array, as one batch entry
        return np.ascontiguousarray(a.reshape((-1,) + per_token)[lo:lo + L])[None]

    q, k = sl(inp.q, (H, inp.dk)), sl(inp.k, (H, inp.dk))
    v, la, be = sl(inp.v, (H, inp.dv)), sl(inp.log_alpha, (H, inp.dk)), sl(inp.beta, (H,))
    s0 = None if inp.initial_state is None else inp.initial_state[n:n + 1]
    _, s = oracle.recurrent(q, k, v, la, be, s0, o_tokens=0)
    return s[0]


def _run(inp, interval, max_snaps, slot_of, num_slots):
    import torch
    from gated_delta_rule_139_b200 import kda_fwd, kda_fwd_snap
    d = to_device(inp)
    slots = torch.tensor(slot_of, dtype=torch.int32, device="cuda").reshape(-1, max_snaps)
    pool = torch.full((num_slots, inp.H, inp.dk, inp.dv), 7.5, device="cuda")
    o, s = kda_fwd_snap(**d, snap_interval=interval, snap_slots=slots, snap_pool=pool)
    o_ref, s_ref = kda_fwd(**d)
    torch.cuda.synchronize()
    # snapshots change no other result
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    return pool.cpu().numpy().astype(np.float64)


def _check_pool(inp, pool, interval, max_snaps, slot_of, tol_abs=None):
    lens = [hi - lo for lo, hi in seq_bounds(inp)]
    used = set()
    for n, L in enumerate(lens):
        for j in range(max_snaps):
            sl = slot_of[n * max_snaps + j]
            if sl < 0 or (j + 1) * interval > L:
                continue
            used.add(sl)
            ref = _prefix_state(inp, n, (j + 1) * interval)
            got = pool[sl]
            if tol_abs is not None:
                assert np.abs(got - ref).max() <= tol_abs, (n, j)
            else:
                for h in range(inp.H):
                    err = np.linalg.norm(got[h] - ref[h]) / np.linalg.norm(ref[h])
                    assert err <= TOL_BF16_REL_FRO, (n, j, h, err)
    for sl in set(range(pool.shape[0])) - used:
        assert (pool[sl] == 7.5).all(), sl


def test_snapshots_tensor_core_path_packed():
    lens = [640, 100, 1000, 0, 64 * 5]
    inp = make_inputs(1, 0, 3, 128, 128, bf16=True, seed=200, seq_lens=lens, state_sigma=0.05,
                      gate_sigma=2.0)
    interval, max_snaps = 128, 8
    rng = np.random.default_rng(0)
    slot_of = list(rng.permutation(40)[:len(lens) * max_snaps])
    slot_of = [int(x) if x % 5 else -1 for x in slot_of]  # some snapshots not requested
    pool = _run(inp, interval, max_snaps, slot_of, 40)
    _check_pool(inp, pool, interval, max_snaps, slot_of)


@pytest.mark.parametrize("seg_chunks", ["1", "3"])
def test_snapshots_with_segment_split(monkeypatch, seg_chunks):
    monkeypatch.setenv("KDA_SEG_CHUNKS", seg_chunks)
    inp = make_inputs(2, 64 * 7 + 9, 2, 128, 128, bf16=True, seed=201, state_sigma=0.05)
    interval, max_snaps = 64, 7
    slot_of = list(range(2 * max_snaps))
    pool = _run(inp, interval, max_snaps, slot_of, 2 * max_snaps)
    _check_pool(inp, pool, interval, max_snaps, slot_of)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64)])
def test_snapshots_cuda_core_path_fp32(dk, dv):
    lens = [64 * 3 + 5, 64 * 2]
    inp = make_inputs(1, 0, 2, dk, dv, bf16=False, seed=202, seq_lens=lens, state_sigma=0.05)
    interval, max_snaps = 64, 4
    slot_of = [3, 0, 5, -1, 1, 2, -1, 4]
    pool = _run(inp, interval, max_snaps, slot_of, 6)
    _check_pool(inp, pool, interval, max_snaps, slot_of, tol_abs=TOL_F32_MAX_ABS)


def test_resume_from_snapshot_bitwise(monkeypatch):
    """Without segment split, the snapshot at 320 tokens is bitwise the final
    state of the first 320 tokens, and resuming from it reproduces the rest."""
    import torch
    from gated_delta_rule_139_b200 import kda_fwd, kda_fwd_snap
    monkeypatch.setenv("KDA_SEG_CHUNKS", "100000")
    inp = make_inputs(1, 640, 2, 128, 128, bf16=True, seed=203, state_sigma=0.05)
    d = to_device(inp)
    slots = torch.tensor([[-1, -1, -1, -1, 0]], dtype=torch.int32, device="cuda")
    pool = torch.zeros(1, 2, 128, 128, device="cuda")
    o, _ = kda_fwd_snap(**d, snap_interval=64, snap_slots=slots, snap_pool=pool)
    keys = ("q", "k", "v", "log_alpha", "beta")
    a = {k_: d[k_][:, :320].contiguous() for k_ in keys}
    b = {k_: d[k_][:, 320:].contiguous() for k_ in keys}
    _, s1 = kda_fwd(**a, initial_state=d["initial_state"])
    o2, _ = kda_fwd(**b, initial_state=pool)
    torch.cuda.synchronize()
    assert torch.equal(pool, s1) and torch.equal(o2, o[:, 320:])


def test_snapshot_slot_out_of_range_sets_status():
    import torch
    from gated_delta_rule_139_b200 import KDAError, check_device, kda_fwd_snap
    inp = make_inputs(1, 256, 1, 128, 128, bf16=True, seed=204)
    d = to_device(inp)
    check_device()
    slots = torch.tensor([[0, 9]], dtype=torch.int32, device="cuda")
    pool = torch.zeros(2, 1, 128, 128, device="cuda")
    kda_fwd_snap(**d, snap_interval=128, snap_slots=slots, snap_pool=pool)
    with pytest.raises(KDAError) as e:
        check_device()
    assert e.value.name == "KDA_ERR_INVALID_ARG"
    assert pool[1].abs().sum().item() == 0 and pool[0].abs().sum().item() > 0
