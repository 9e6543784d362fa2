"""The failure path of the kernels' bounded device waits, made to run on purpose.

Every wait of the tensor-core kernels on an mbarrier is bounded in wall time: when
the bound passes, the kernel records KDA_ERR_DEVICE_TIMEOUT in the device status
word and returns.  kda_selftest_wait runs that same wait on an mbarrier nothing
arrives at (a 1 ms bound here), so the wait gives up by itself -- no fault, no
hang -- and the host must see the timeout once, then a clean status, and the
context must stay usable for a forward pass that matches the oracle.
"""
import time

import numpy as np
import pytest

import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, rel_fro_per_head, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_a_timeout():
    import gated_delta_rule_139_b200 as kda
    lib = kda.load_library()
    kda.check_device()  # start from a clean status word
    t0 = time.perf_counter()
    assert lib.kda_selftest_wait(1_000_000, 0, None) == 0  # 1 ms, nothing arrives
    with pytest.raises(kda.KDAError) as err:
        kda.check_device()
    elapsed = time.perf_counter() - t0
    assert "KDA_ERR_DEVICE_TIMEOUT" in str(err.value)
    assert elapsed < 5.0, elapsed  # the wait gave up after its bound
    kda.check_device()  # reading the status cleared it
    # the same wait with the arrival made: no timeout
    assert lib.kda_selftest_wait(1_000_000, 1, None) == 0
    kda.check_device()
    # out-of-range bounds are argument errors
    assert kda.STATUS[lib.kda_selftest_wait(10, 0, None)] == "KDA_ERR_INVALID_ARG"
    assert kda.STATUS[lib.kda_selftest_wait(10 ** 9, 0, None)] == "KDA_ERR_INVALID_ARG"


def test_forward_runs_clean_after_a_timeout():
    import gated_delta_rule_139_b200 as kda
    lib = kda.load_library()
    assert lib.kda_selftest_wait(1_000_000, 0, None) == 0
    with pytest.raises(kda.KDAError):
        kda.check_device()
    inp = make_inputs(1, 64 * 5 + 9, 2, 128, 128, bf16=True, seed=44, state_sigma=0.05)
    o_g, s_g = run_gpu(inp)
    kda.check_device()  # the forward pass itself recorded nothing
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)
    eo, es = rel_fro_per_head(o_g, o_r, s_g, s_r, inp)
    assert np.isfinite(o_g).all()
    assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
