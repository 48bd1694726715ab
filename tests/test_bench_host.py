"""Host-side pieces of bench.py that need no GPU: the source hash that ties the
committed DRAM-traffic summary to the kernel code it was captured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_hash_ignores_comments_and_layout_only():
    src = "int f(int a) {  // add one\n  return a + 1; /* the\n  answer */ }\n"
    same = "int f(int a)\n{\n    return a + 1;   // comment moved\n}\n"
    other = "int f(int a) { return a + 2; }\n"
    assert bench._code_only(src) == bench._code_only(same)
    assert bench._code_only(src) != bench._code_only(other)


def test_traffic_summary_matches_or_is_null():
    # the summary is used only when its hash equals the current sources'; otherwise null
    t = bench.ncu_traffic("gateup_prefill_large")
    import json
    d = json.load(open(bench.TRAFFIC_FILE))
    if d["csrc_hash"] == bench.csrc_hash():
        assert t == d["kernels"]["gateup_prefill_large"]["dram_bytes_per_launch"]
    else:
        assert t is None


def test_peaks_prefer_the_measured_file(tmp_path, monkeypatch):
    # the measured peaks file, when present, supplies both GEMM figures; without it the
    # stated fallback applies and no sustained figure is claimed
    import json
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    pk, kind = bench.peaks()
    assert kind == "measured" and pk["bf16_tflops_sustained"] == 1300.0 and pk["hbm_gbs"] == 6000.0
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    pk, kind = bench.peaks()
    assert kind == "fallback" and pk == bench.FALLBACK_PEAKS and "bf16_tflops_sustained" not in pk
