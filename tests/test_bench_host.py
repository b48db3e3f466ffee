"""Host-side helpers of bench.py: the algorithmic work it divides by (against brute-force
sums from the definitions), the source hash that keys the committed DRAM traffic (a kernel
variant shares its file's hash; an edited file loses its traffic figure), and the
contract keys of the reference arm's JSON line."""
import json

import bench


def test_algorithmic_work_matches_brute_force():
    T, k = 300, 64
    w = bench.algorithmic_work(T, k)
    pairs = sum(t + 1 for t in range(T))
    sel = sum(min(t + 1, k) for t in range(T))
    assert w["indexer_flop"] == 2 * 16 * 64 * pairs
    assert w["mla_flop"] == 2 * 16 * (576 + 512) * sel
    assert w["mla_gather_bytes"] == 1152 * sel
    assert bench.algorithmic_work(T, k, kv_bytes=1)["mla_gather_bytes"] == 576 * sel
    assert w["topk_read_bytes"] == 4 * pairs


def test_traffic_keyed_by_source_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash("mla_mma.cu")
    assert h == bench.kernel_source_hash("mla_mma.cu:fp8")
    assert h != bench.kernel_source_hash("topk.cu")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({
        "mla_mma.cu": {"source_hash": "aaa", "bytes_per_launch_full": 123},
        "topk.cu": {"source_hash": "stale", "bytes_per_launch_full": 456}}))
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda name: {"mla_mma.cu": "aaa", "topk.cu": "new"}[name.split(":")[0]])
    assert bench.load_traffic("mla_mma.cu") == 123
    assert bench.load_traffic("topk.cu") is None        # edited since the capture
    assert bench.load_traffic("mla_mma.cu:fp8") is None  # never captured


def test_reference_line_keys(monkeypatch):
    """The reference arm's JSON line (CPU oracle), on a tiny stand-in workload."""
    from sparse_attention_17_b200 import inputs as G
    monkeypatch.setattr(bench, "make_inputs", lambda T, k, seed, kv_dtype="bf16":
                        G.mla_prefill_gauss(T=256, seed=seed, k=64))

    class A:
        T, topk, steps, warmup, cpu_seconds = 256, 64, 1, 0, 0.2

    line = bench.run_reference(A, 0, 1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "impl", "config", "cpu_baseline",
                "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert bench.run_reference(A, 1, 2) is None  # only rank 0 runs the oracle


def test_tensor_peak_follows_the_clock_record():
    """Burst peak when the timed region ran at the maximum SM clock without a power cap;
    sustained otherwise (a kernel timed under the power cap)."""
    peaks = {"bf16_tflops": 1646.6, "bf16_tflops_sustained": 1407.5}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1342.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.choose_tensor_peak(peaks, at_max)[0] == 1646.6
    assert bench.choose_tensor_peak(peaks, capped)[0] == 1407.5
    assert bench.choose_tensor_peak(peaks, slow)[0] == 1407.5
    assert bench.choose_tensor_peak({"bf16_tflops": 1590.0}, capped)[0] == 1590.0
    unsampled = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
    assert bench.choose_tensor_peak(peaks, unsampled)[0] == 1407.5


def test_reference_line_marks_extrapolated_step(monkeypatch):
    from sparse_attention_17_b200 import inputs as G
    monkeypatch.setattr(bench, "make_inputs", lambda T, k, seed, kv_dtype="bf16":
                        G.mla_prefill_gauss(T=256, seed=seed, k=64))

    class A:
        T, topk, steps, warmup, cpu_seconds = 256, 64, 1, 0, 0.2

    line = bench.run_reference(A, 0, 1)
    assert line["extrapolated"] is True and line["sampled_ms_per_step"] > 0
