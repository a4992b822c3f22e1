"""bench.py's host arithmetic on CPU: the roofline of the dominant stage
(achieved = algorithmic work × steps ÷ device time, against the measured
peak), the committed DRAM traffic lookup (only while the profiled source
region is unchanged), the whole-job throughput and the bounded correlation
stage's byte model."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6553.0, "bf16_tflops": 1641.0, "bf16_tflops_sustained": 1389.0, "sm_max_mhz": 1965.0,
         "source": "measured"}


def test_roofline_of_the_dominant_stage_by_hand():
    stages = {"rows": {"ms": 200.0, "launches": 400}, "nnls": {"ms": 150.0, "launches": 100},
              "solve": {"ms": 10.0, "launches": 20}, "gram": {"ms": 0.0, "launches": 0}}
    models = {"rows": {"bound": "hbm", "bytes": 3.0e9}, "solve": {"bound": "fp64", "flops": 1.0e10}}
    traffic = {"rows": {"bytes_per_launch": 8.0e6, "source": "profiles/x.md"}}
    rf = bench.roofline(stages, 4, models, PEAKS, {"sm_mhz": 1900.0}, traffic)
    assert rf["kernel"] == "rows"                            # the most device time
    assert rf["launches_per_step"] == 100 and rf["avg_launch_ms"] == 0.5
    # 3 GB per step, 4 steps, 0.2 s of stage time: 60 GB/s
    assert abs(rf["achieved"] - 60.0) < 1e-9 and rf["unit"] == "GB/s"
    assert abs(rf["frac"] - 60.0 / 6553.0) < 1e-12
    assert rf["traffic"] == 8.0e6 and rf["traffic_source"] == "profiles/x.md"
    assert list(rf["all_stages"]) == ["rows", "nnls", "solve"]   # by device time; unused stages left out
    assert rf["all_stages"]["nnls"]["bound"] is None             # no model: no fraction claimed
    # fp64 stage: 1e10 flops × 4 steps / 10 ms = 4 TFLOP/s against 148 × 64 × 2 × 1.9 GHz
    s = rf["all_stages"]["solve"]
    assert s["bound"] == "alu" and abs(s["achieved"] - 4.0) < 1e-9
    assert abs(s["frac"] - 4.0 / (148 * 64 * 2 * 1900e6 / 1e12)) < 1e-12


def test_traffic_without_a_committed_entry_is_null():
    stages = {"nnls": {"ms": 5.0, "launches": 10}}
    rf = bench.roofline(stages, 1, {"nnls": {"bound": "hbm", "bytes": 1e6}}, PEAKS, None, {})
    assert rf["traffic"] is None and "traffic_source" not in rf


def test_committed_traffic_follows_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("head\n// begin --\nkernel body\n// end --\ntail\n")
    import hashlib
    region = src.read_text()[src.read_text().index("// begin --"):src.read_text().index("// end --")]
    rec = {"rows": {"workload": "w1", "stage": "rows", "source": "k.cu", "region_begin": "// begin --",
                    "region_end": "// end --", "region_sha256_16": hashlib.sha256(region.encode()).hexdigest()[:16],
                    "dram_bytes_per_launch": 123.0, "summary": "profiles/k.md"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.committed_traffic("w1") == {"rows": {"bytes_per_launch": 123.0, "source": "profiles/k.md"}}
    assert bench.committed_traffic("w2") == {}                # another workload
    src.write_text("head\n// begin --\nkernel body changed\n// end --\ntail\n")
    assert bench.committed_traffic("w1") == {}                # the kernel changed since the capture


def test_the_committed_rows_traffic_matches_the_current_source():
    """The entry bench.py uses for the model's dominant stage still hashes to
    the bounded pass as it stands (a change to k_gbound / k_rows nulls it)."""
    got = bench.committed_traffic("qwen3_4b_model_H288_T8192_n8192_d128_lognormal")
    assert "rows" in got and got["rows"]["bytes_per_launch"] > 0


def test_job_throughput_and_max_over_ranks():
    assert bench.job_throughput(288, 1, 131.0) == 288 / 0.131
    assert bench.job_throughput(288, 4, 131.0) == 4 * 288 / 0.131    # weak scaling: all ranks' heads
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5


def test_bounded_stage_byte_model_by_hand():
    from attention_matching_b200 import workloads as W
    wl = W.Workload("w", [], [8, 20], 4, 2, "bf16")
    n, T, d = 8192, 8192, 128
    ldn = n
    m = bench.stage_models(wl, n, [T, T], d, ldn, "bounded", 100, True)
    # rows: 100 evaluated rows of ldn fp32, plus per key and pass its 64 group norms, the bound and the flag
    passes = (8 + 7) // 8 + (20 + 7) // 8
    assert m["rows"]["bytes"] == 100 * ldn * 4 + passes * T * (64 * 4 + 8)
    assert m["rows"]["bound"] == "hbm"
