"""Child process of test_debug_build_gpu.py: runs with KDA_LIBRARY pointing at the
debug build (-DKDA_DEBUG) and prints one JSON line of findings."""
import json
import sys

import numpy as np
import torch

import gated_delta_rule_139_b200 as kda
import oracle
from gated_delta_rule_139_b200.inputs import make_inputs
from kda_testlib import rel_fro_per_chunk, rel_fro_per_head, run_gpu, to_device

res = {"library": kda.library_path}


def status():
    try:
        kda.check_device()
        return "ok"
    except kda.KDAError as e:
        return str(e)


# valid segmented and packed forward passes: no check fires, every guard band holds
for name, inp in (
        ("segmented", make_inputs(2, 4096, 4, 128, 128, bf16=True, seed=61, state_sigma=0.02,
                                  gate_sigma=2.0)),
        ("packed", make_inputs(1, 0, 4, 128, 128, bf16=True, seed=62, state_sigma=0.02,
                               seq_lens=[700, 0, 2100, 64, 33, 1200]))):
    o, s = run_gpu(inp)
    res[name + "_launches"] = kda.last_launch_count()
    res[name + "_status"] = status()
    o_r, s_r = oracle.recurrent(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.initial_state,
                                inp.cu_seqlens)
    res[name + "_err"] = list(rel_fro_per_head(o, o_r, s, s_r, inp))
    res[name + "_err_chunk"] = rel_fro_per_chunk(o, o_r, inp)[0]

# a span whose workspace segment table has entry 1 (sequence 0, second segment)
# ending past its sequence: the forward pass's index check catches it
inp = make_inputs(2, 64 * 40, 2, 128, 128, bf16=True, seed=63, state_sigma=0.02)
d = to_device(inp)
ws = kda.span_workspace(d["k"])
kda.kda_span_transition(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws)
torch.cuda.synchronize()
res["span_transition_status"] = status()
ent = ws[40:80].cpu().numpy().view(np.int64)  # t_begin, t_end, (n, j), (last, pad), c_base
res["entry1"] = [int(ent[0]), int(ent[1])]
bad = ws[40:80].clone()
bad.view(torch.int64)[1] = 64 * 40 + 64  # past the end of sequence 0
ws[40:80] = bad
kda.kda_span_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], ws, d["initial_state"])
torch.cuda.synchronize()
res["corrupt_status"] = status()
# the context stays usable: the next call runs clean
inp2 = make_inputs(1, 64 * 3 + 5, 2, 128, 128, bf16=True, seed=64)
run_gpu(inp2)
res["after_status"] = status()
print(json.dumps(res))
sys.stdout.flush()
