"""Host logic of bench.py's roofline denominators and DRAM-traffic records
(no GPU): the measured peaks file is read key by key with the fallback
figures behind it, and a committed ncu traffic record counts only for its
own workload and kernel, and only while that kernel's sources are the ones
it was captured on."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_fallback_peaks_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert peaks == bench.FALLBACK_PEAKS
    assert src.startswith("fallback")


def test_measured_peaks_fill_missing_keys_from_the_fallback(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6540.2, "bf16_tflops": 1631.7}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src.startswith("measured")
    assert peaks["hbm_gbs"] == 6540.2 and peaks["bf16_tflops"] == 1631.7
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]


def test_committed_traffic_records_are_well_formed():
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    assert d["records"]
    for r in d["records"]:
        assert r["kind"] in bench.KERNEL_SOURCES
        assert r["dram_bytes_per_launch"] == r["dram_read"] + r["dram_write"] > 0
        assert "ncu " in r["command"] and "--clock-control none" in r["command"]


def _fake_tree(tmp_path, body):
    csrc = tmp_path / "mixture_experts_layer_56_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("gemm_sm100_pair.cu", "gemm_sm100.h", "gemm_sm100.cu", "sm100_ptx.cuh",
                 "common.cuh", "decode_fused.cu", "kernels.cu"):
        (csrc / name).write_text(body.get(name, name))
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_record_follows_its_own_kernel_sources(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, {})
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash("gate_up")
    rec = {"kind": "gate_up", "workload": "large", "source_hash": h, "dram_read": 7,
           "dram_write": 3, "dram_bytes_per_launch": 10}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({"records": [rec]}))
    assert bench.ncu_traffic("large") == 10
    assert bench.ncu_traffic("small") is None              # another workload
    assert bench.ncu_traffic("large", "decode_layer") is None  # another kernel
    # a file outside the gate/up kernel's sources changes nothing
    (csrc / "kernels.cu").write_text("changed")
    (csrc / "gemm_sm100.cu").write_text("changed")          # the single-CTA kernel
    assert bench.ncu_traffic("large") == 10
    # comments and blank lines are not the kernel
    (csrc / "gemm_sm100_pair.cu").write_text("// a note\ngemm_sm100_pair.cu  /* more */\n\n")
    assert bench.ncu_traffic("large") == 10
    # a change to the CTA-pair kernel's code voids the record
    (csrc / "gemm_sm100_pair.cu").write_text("changed")
    assert bench.ncu_traffic("large") is None
