"""kda_fwd_noalloc: the entry point for callers that cannot allocate device
memory (its temporaries live in a fixed scratch array inside the library).

Checked through the C ABI against the ordinary kda_fwd entry point, twice in a
row (the scratch array keeps the previous call's contents), within the bf16
tolerance of the parity tests.  This file sorts last so that a run stopping at
its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_139_b200 as kda
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, TOL_F32_MAX_ABS, out_to_f64, rel_fro_per_head, to_device

pytestmark = pytest.mark.gpu


def _both(inp):
    import torch
    d = to_device(inp)
    o_ref, s_ref = kda.kda_fwd(**d)
    torch.cuda.synchronize()
    runs = []
    for _ in range(2):
        o, s = kda.kda_fwd_noalloc(**d)
        torch.cuda.synchronize()
        assert kda.last_launch_count() > 0
        runs.append((out_to_f64(o), s.cpu().numpy().astype(np.float64)))
    return (out_to_f64(o_ref), s_ref.cpu().numpy().astype(np.float64)), runs


@pytest.mark.parametrize("case", ["segmented", "packed", "fp32"])
def test_noalloc_matches_kda_fwd_two_calls(case):
    if case == "segmented":  # 64 chunks per sequence: cut into segments
        inp = make_inputs(2, 4096, 8, 128, 128, bf16=True, seed=41, state_sigma=0.02,
                          gate_sigma=2.0)
    elif case == "packed":
        inp = make_inputs(1, 0, 4, 128, 128, bf16=True, seed=42, state_sigma=0.02,
                          seq_lens=[1000, 0, 3000, 64, 17])
    else:
        inp = make_inputs(1, 300, 2, 64, 64, bf16=False, seed=43)
    (o_ref, s_ref), runs = _both(inp)
    for o, s in runs:
        assert np.isfinite(o).all() and np.isfinite(s).all()
        if inp.bf16:
            eo, es = rel_fro_per_head(o, o_ref, s, s_ref, inp)
            assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
        else:
            assert np.abs(o - o_ref).max() <= TOL_F32_MAX_ABS
            assert np.abs(s - s_ref).max() <= TOL_F32_MAX_ABS


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
