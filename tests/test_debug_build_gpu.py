"""Debug aids: the -DKDA_DEBUG build's device index checks and workspace guard
bands, and guard bands around a caller-owned span workspace.

The debug build runs in a child process (tests/debug_build_child.py) that loads
_build/debug/libkda.so through KDA_LIBRARY; it is built here when missing.  In it:
segmented and packed forward passes match the oracle with a clean device status
(no index check fires on valid tables; the guard bands around every buffer of
kda_fwd's workspace keep their fill pattern), and a span forward pass whose
workspace segment table has one entry moved past its sequence's end reports the
failed index check through kda_check_device -- the block returns before any
access through that entry -- after which the next call runs clean.

With the release library, a span workspace placed between two 64 KiB guard bands
of a larger buffer: kda_span_transition and kda_span_forward write inside it
only, for a segmented span and for one that is a single segment.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import gated_delta_rule_139_b200 as kda
import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import TOL_BF16_REL_FRO, TOL_BF16_REL_FRO_CHUNK, rel_fro_per_head, to_device

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def debug_run():
    from gated_delta_rule_139_b200 import build as kda_build
    lib = kda_build.build(variant="debug")
    env = dict(os.environ, KDA_LIBRARY=lib,
               PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests")]))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_child.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["library"] == lib
    return res


@pytest.mark.parametrize("case", ["segmented", "packed"])
def test_debug_build_valid_inputs_run_clean(debug_run, case):
    assert debug_run[case + "_launches"] == 4  # segment table, pass 1, scan, pass 3
    assert debug_run[case + "_status"] == "ok"
    eo, es = debug_run[case + "_err"]
    assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
    assert debug_run[case + "_err_chunk"] <= TOL_BF16_REL_FRO_CHUNK


def test_debug_build_index_check_catches_a_bad_segment_entry(debug_run):
    assert debug_run["span_transition_status"] == "ok"
    assert debug_run["entry1"] == [512, 1024]  # 8-chunk segments of a 40-chunk sequence
    assert "index check failed" in debug_run["corrupt_status"], debug_run["corrupt_status"]
    assert debug_run["after_status"] == "ok"


@pytest.mark.parametrize("T", [64 * 40 + 17, 64 * 6])
def test_span_workspace_writes_stay_inside_it(T):
    import torch
    inp = make_inputs(2, T, 2, 128, 128, bf16=True, seed=65, state_sigma=0.02)
    d = to_device(inp)
    n = kda.span_workspace(d["k"]).numel()
    G = 64 << 10
    buf = torch.full((G + n + G,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + n]
    assert ws.data_ptr() % 256 == 0
    kda.kda_span_transition(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws)
    o, s = kda.kda_span_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws,
                                d["initial_state"])
    torch.cuda.synchronize()
    kda.check_device()
    assert bool((buf[:G] == 0xA5).all()) and bool((buf[G + n:] == 0xA5).all())
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state)
    eo, es = rel_fro_per_head(o.float().cpu().numpy().astype(np.float64), o_r,
                              s.cpu().numpy().astype(np.float64), s_r, inp)
    assert eo <= TOL_BF16_REL_FRO and es <= TOL_BF16_REL_FRO, (eo, es)
