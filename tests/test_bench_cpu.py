"""Host-side helpers of bench.py: the committed DRAM-traffic record is reported
only for the workload and the kernel sources it was captured on, and pass 1's
algorithmic bytes follow the library's segment plan."""
import hashlib
import json
import os
import types

import bench


def _inp(T, H, B=1):
    return types.SimpleNamespace(T=T, H=H, B=B, dk=128, dv=128, cu_seqlens=None, n_seqs=B,
                                 tokens=B * T, seq_lens=[T] * B)


def test_traffic_record_needs_the_same_workload_and_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles").mkdir()
    rec = {"tc_pass1_transitions": {"bytes_per_launch": 5.0e9, "sources": ["k.cu"], "sha256": sha,
                                    "workload": "prefill_1m"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("tc_pass1_transitions", "prefill_1m") == 5.0e9
    assert bench.recorded_traffic("tc_pass1_transitions", "prefill_64k") is None
    assert bench.recorded_traffic("tc_pass3_forward", "prefill_1m") is None
    src.write_text("kernel v2")  # the kernel changed after the capture
    assert bench.recorded_traffic("tc_pass1_transitions", "prefill_1m") is None


def test_committed_traffic_record_names_its_workload():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for tag, r in rec.items():
        assert r["workload"] == "prefill_1m" and r["bytes_per_launch"] > 0, tag


def test_pass1_algorithmic_bytes_follow_the_segment_plan():
    inp = _inp(1 << 20, 8)  # the 1M-token prefill: 37 segments of 443 chunks per head
    seg, cut = bench.segment_plan(inp)
    assert cut and seg == 443
    segs = -(-16384 // seg)
    # pass 1 reads q, k, v (bf16), log alpha and beta (fp32) of every token once and
    # writes one (B, M) pair per segment with a successor and head
    per_tok = 8 * (128 * 2 * 3 + 128 * 4 + 4)
    want = 16384 * 64 * per_tok + (segs - 1) * 8 * 2 * 128 * 128 * 4
    assert bench.kernel_algorithmic_bytes("tc_pass1_transitions", inp, 123) == want
    assert bench.kernel_algorithmic_bytes("tc_pass3_forward", inp, 123) == 123
    assert bench.kernel_algorithmic_bytes("tc_pass1_transitions", _inp(64 * 4, 8), 1) == 0
