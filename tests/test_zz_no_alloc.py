"""kda_fwd_noalloc: the entry point for callers that cannot allocate device
memory (its temporaries live in a fixed 32 MiB scratch array inside the library).

Each case runs it twice in a row through the C ABI (the scratch array keeps the
previous call's contents) and checks both results against the fp64 oracle, per
(sequence, head) and per 64-token chunk within the bf16 tolerances of the parity
tests, and, as a second check, against the ordinary kda_fwd entry point.  Two
cases have a default segment plan whose temporaries exceed the scratch array,
so the entry point coarsens the plan: once to longer segments, once to a single
segment per sequence (visible as two kernel launches instead of four).  This
file sorts last so that a run stopping at its first failure has already run every
other test; it needs no state left by them.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_139_b200 as kda
import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import (TOL_BF16_REL_FRO, TOL_BF16_REL_FRO_CHUNK, TOL_F32_MAX_ABS, out_to_f64,
                         rel_fro_per_chunk, rel_fro_per_head, to_device)

pytestmark = pytest.mark.gpu

# (B, T, H, d, bf16, extra make_inputs arguments, launches of kda_fwd_noalloc or None)
CASES = {
    # 64 chunks per sequence: cut into segments, temporaries well inside the scratch
    "segmented": (2, 4096, 8, 128, True, dict(seed=41, state_sigma=0.02, gate_sigma=2.0), 4),
    "packed": (1, 0, 4, 128, True, dict(seed=42, state_sigma=0.02, seq_lens=[1000, 0, 3000, 64, 17]), 4),
    "fp32": (1, 300, 2, 64, False, dict(seed=43), None),
    # default plan: 29-chunk segments, about 63 MB of transitions and incoming states;
    # coarsened to 116-chunk segments (25 MB), still cut
    "coarsened": (1, 16384, 32, 128, True, dict(seed=44, state_sigma=0.02), 4),
    # default plan: 22-chunk segments (75 MB); 44-chunk segments still overflow
    # (57 MB), so the sequence becomes one segment and only the segment table is kept
    "one_segment": (1, 4096, 96, 128, True, dict(seed=45, state_sigma=0.02), 2),
}


def _runs(inp):
    import torch
    d = to_device(inp)
    o_fwd, s_fwd = kda.kda_fwd(**d)
    torch.cuda.synchronize()
    fwd_launches = kda.last_launch_count()
    runs = []
    for _ in range(2):
        o, s = kda.kda_fwd_noalloc(**d)
        torch.cuda.synchronize()
        launches = kda.last_launch_count()
        runs.append((out_to_f64(o), s.cpu().numpy().astype(np.float64), launches))
    return (out_to_f64(o_fwd), s_fwd.cpu().numpy().astype(np.float64), fwd_launches), runs


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_the_oracle_two_calls(case):
    B, T, H, dd, bf16, kw, want_launches = CASES[case]
    inp = make_inputs(B, T, H, dd, dd, bf16=bf16, **kw)
    (o_fwd, s_fwd, fwd_launches), runs = _runs(inp)
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                inp.cu_seqlens)
    for o, s, launches in runs:
        assert launches > 0
        if want_launches is not None:
            assert launches == want_launches, (launches, fwd_launches)
        assert np.isfinite(o).all() and np.isfinite(s).all()
        if inp.bf16:
            eo, es = rel_fro_per_head(o, o_r, s, s_r, inp)
            assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
            ec, where = rel_fro_per_chunk(o, o_r, inp)
            assert ec <= TOL_BF16_REL_FRO_CHUNK, (ec, where)
            # the ordinary entry point on the same inputs
            eo, es = rel_fro_per_head(o, o_fwd, s, s_fwd, inp)
            assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
        else:
            assert np.abs(o - o_r).max() <= TOL_F32_MAX_ABS
            assert np.abs(s - s_r).max() <= TOL_F32_MAX_ABS
            assert np.abs(o - o_fwd).max() <= TOL_F32_MAX_ABS
    if case == "one_segment":
        assert fwd_launches == 4  # kda_fwd itself cuts the sequence


def test_noalloc_rejects_a_table_larger_than_the_scratch():
    import torch
    N = 2_000_000  # zero-length sequences: the segment table alone needs > 32 MiB
    cu = torch.zeros(N + 1, dtype=torch.int32, device="cuda")
    d = kda.Dims(1, 0, 1, 128, 128, N, kda.KDA_BF16)
    lib = kda.load_library()
    rc = lib.kda_fwd_noalloc(None, None, None, None, None, None, ctypes.c_void_p(cu.data_ptr()),
                             64, None, None, ctypes.byref(d), None)
    assert kda.STATUS[rc] == "KDA_ERR_UNSUPPORTED"
    assert "scratch" in lib.kda_last_error().decode()
    assert kda.last_launch_count() == 0
