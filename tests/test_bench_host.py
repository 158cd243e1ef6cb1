"""Host-side pieces of bench.py, on the CPU.

* A committed traffic summary is attached to a bench line only when it was
  taken on the current kernel source and on a call of about the same
  algorithmic bytes (within 5%: later decode states are a few tokens longer;
  a smaller --batch of the same workload gets none).
* The oracle timing samples whole sequences or (sequence, KV head) units and
  reports bytes over seconds either way.
"""

import os
import shutil

import numpy as np
import pytest

import bench


def test_traffic_attached_only_to_a_call_of_the_captured_size():
    full = bench.profiled_traffic("long16")
    assert full is not None and full > 4.29e9
    alg = full / 1.0029
    assert bench.profiled_traffic("long16", algorithmic=alg) == full
    assert bench.profiled_traffic("long16", algorithmic=alg * 1.02) == full  # later states
    assert bench.profiled_traffic("long16", algorithmic=alg / 4) is None   # batch 2 of 8


def test_traffic_ignored_when_the_kernel_source_changed(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), prof)
    path = prof / "decode_long16_traffic.txt"
    text = path.read_text()
    stale = "\n".join(("kernel_source_sha256_16: 0000000000000000"
                       if line.startswith("kernel_source_sha256_16:") else line)
                      for line in text.splitlines())
    path.write_text(stale + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("long16") is None


@pytest.mark.parametrize("per_kv_head", [False, True])
def test_oracle_timing_units(per_kv_head):
    w = bench.make_workload("gqa", 0, 4)
    gbs, seqs_per_s, desc, secs = bench.time_oracle(w, 0.05, per_kv_head=per_kv_head)
    assert gbs > 0 and seqs_per_s > 0 and secs > 0
    assert ("(sequence, KV head) units" in desc) == per_kv_head
    assert "float64 NumPy oracle, 1 thread" in desc
