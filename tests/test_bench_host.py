"""Host-side pieces of bench.py that feed the reported numbers: the algorithmic
byte counts behind every roofline fraction, the clock-sample parser that decides
whether a run is kept, the peak lookup and the counter gate on `traffic`."""
import hashlib
import json

import bench


def test_algorithmic_bytes_of_the_headline_workload():
    ab = bench.algorithmic_bytes_per_query(131072)
    # every causal index key once (256 B), the query's indexer matrix and weights,
    # 2048 gathered latent rows of 1152 B, q, gate, the fp32 output and the indices
    assert ab["k_idx"] == 131072 * 256
    assert ab["indexer"] == 131072 * 256 + 64 * 128 * 2 + 64 * 2 == 33_570_944
    assert ab["kv_rows"] == 2048 * 576 * 2
    assert ab["total"] == 36_143_360
    # 32 queries: the indexer's bytes per launch quoted with the roofline
    assert 32 * ab["indexer"] == 1_074_270_208


def test_algorithmic_bytes_with_e4m3_keys():
    ab = bench.algorithmic_bytes_per_query(131072, key_bytes=1)
    assert ab["k_idx"] == 131072 * 128 and ab["q_idx"] == 64 * 128
    assert ab["total"] == 19_357_952
    # only the indexer's operands shrink
    full = bench.algorithmic_bytes_per_query(131072)
    assert full["total"] - ab["total"] == 131072 * 128 + 64 * 128


def _sampler_with(lines):
    s = bench.ClockSampler(0)
    s.lines = lines
    return s.summary()


def test_clock_summary_reads_reasons_and_median():
    row = "0, {sm}, 1965, 900.5, 0x0000000000000004, {hw}, Not Active, {swt}, {cap}"
    lines = [row.format(sm=1965, hw="Not Active", swt="Not Active", cap="Active"),
             row.format(sm=1900, hw="Not Active", swt="Not Active", cap="Not Active"),
             row.format(sm=1950, hw="Not Active", swt="Not Active", cap="Not Active")]
    got = _sampler_with(lines)
    assert got["sm_mhz"] == 1950 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["reasons"] == ["sw_power_cap"]
    lines.append(row.format(sm=1200, hw="Active", swt="Active", cap="Not Active"))
    assert _sampler_with(lines)["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_says_so():
    got = _sampler_with([])
    assert got["sm_mhz"] is None and got["reasons"] == ["nvidia-smi unavailable"]
    # malformed rows are skipped, not misread
    assert _sampler_with(["garbage", "0, N/A, 1965, 1, 0x0, x, x, x, x"])["sm_mhz"] is None


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6554.6}))
    assert bench.measured_peaks() == (6554.6, "measured")


def test_traffic_is_reported_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_gated_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("kernel v1")
    entry = {"source_sha256": hashlib.sha256(b"kernel v1").hexdigest(), "dram_bytes_per_launch": 1.0}
    (tmp_path / "profiles" / "counters.json").write_text(json.dumps({"k.cu": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_counters("k.cu")["dram_bytes_per_launch"] == 1.0
    src.write_text("kernel v2")
    assert bench.kernel_counters("k.cu") is None
    assert bench.kernel_counters("missing.cu") is None


def test_causal_indexer_flops_of_the_prefill_chunk():
    # 4096 queries at positions 126,976..131,071: 2 * 64 * 128 * sum(t + 1) = 8.66 TFLOP
    positions = range(126976, 131072)
    assert bench.causal_index_flops(positions) == 2 * 64 * 128 * 4096 * (126977 + 131072) / 2
    assert abs(bench.causal_index_flops(positions) / 1e12 - 8.659) < 1e-3
    assert bench.causal_index_flops([0]) == 2 * 64 * 128


def test_tensor_peak_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_tensor_peak() == (bench.FALLBACK_BF16_TFLOPS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6554.6, "bf16_tflops": 1591.5}))
    assert bench.measured_tensor_peak() == (1591.5, "measured")
