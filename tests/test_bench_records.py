"""bench.py's recorded ncu figures (no GPU): the committed DRAM traffic of the
attention kernel and of the quantizer is reported only while the source it
was captured on is unchanged (else the bench line carries null), and only for
the workload it belongs to."""
import importlib.util
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_committed_records_are_well_formed(bench):
    for name in ("attn_traffic.json", "quant_traffic.json"):
        rec = json.load(open(os.path.join(ROOT, "profiles", name)))
        assert len(rec["kernel_hash"]) == 16
    a = json.load(open(os.path.join(ROOT, "profiles", "attn_traffic.json")))
    assert a["bytes_per_launch"] > a["dram_read_bytes"] + a["dram_write_bytes"] > 0
    q = json.load(open(os.path.join(ROOT, "profiles", "quant_traffic.json")))
    assert q["bytes_per_call"] == sum(q["dram_read_bytes"]) + sum(q["dram_write_bytes"])
    # a record whose source hash matches is what the bench reports
    if a["kernel_hash"] == bench.kernel_hash():
        assert bench.recorded_traffic()["bytes_per_launch"] == a["bytes_per_launch"]
    if q["kernel_hash"] == bench.quant_kernel_hash():
        assert bench.recorded_quant_traffic(q["workload"])["bytes_per_call"] == q["bytes_per_call"]


def test_quant_record_is_per_workload(bench):
    assert bench.recorded_quant_traffic("video480p_b1h12_n32760_d128") is None


def test_records_are_dropped_when_the_source_changes(bench, tmp_path, monkeypatch):
    # a copy of the tree whose profiles name another source hash
    prof = tmp_path / "profiles"
    prof.mkdir()
    for name in ("attn_traffic.json", "quant_traffic.json"):
        rec = json.load(open(os.path.join(ROOT, "profiles", name)))
        rec["kernel_hash"] = "0" * 16
        (prof / name).write_text(json.dumps(rec))
    csrc = tmp_path / "bit_quantized_attention_sage_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("attn.cu", "attn.cuh", "sm100.cuh", "quant.cu", "quant.cuh"):
        (csrc / f).write_bytes(
            open(os.path.join(ROOT, "bit_quantized_attention_sage_b200", "csrc", f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic() is None
    assert bench.recorded_quant_traffic("video720p_b1h40_n75600_d128") is None
