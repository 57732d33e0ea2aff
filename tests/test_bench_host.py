"""Host-side helpers of bench.py, on the CPU: the DRAM-traffic lookup keyed on the
kernel's source and the captured workload, the rotation over input sets that
keeps each step's inputs out of L2, and the peaks' fallback."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _traffic_file(tmp_path, kernel, sha, workload_key, nbytes):
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({kernel: {"dram_bytes_per_launch": nbytes, "source_sha": sha,
                                      "workload_key": workload_key}}))
    return str(f)


def test_traffic_reported_for_the_captured_source_and_workload(tmp_path, monkeypatch):
    k = "kpool_compress"
    sha = bench.kernel_source_sha(bench.STAGE_SOURCE[k])
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _traffic_file(tmp_path, k, sha, "batched", 1234.0))
    assert bench.traffic_for(k, bench.STAGE_SOURCE[k], "batched") == 1234.0
    # another workload, another kernel, or a source changed since the capture: none
    assert bench.traffic_for(k, bench.STAGE_SOURCE[k], "long") is None
    assert bench.traffic_for("indexer", bench.STAGE_SOURCE["indexer"], "batched") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _traffic_file(tmp_path, k, "0" * 16, "batched", 1.0))
    assert bench.traffic_for(k, bench.STAGE_SOURCE[k], "batched") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.json"))
    assert bench.traffic_for(k, bench.STAGE_SOURCE[k], "batched") is None


def test_source_hash_covers_the_shared_header_and_the_kernel():
    a = bench.kernel_source_sha("kpool_compress.cuh")
    assert a == bench.kernel_source_sha("kpool_compress.cuh") and len(a) == 16
    assert a != bench.kernel_source_sha("sparse_mla.cuh")
    assert set(bench.STAGE_SOURCE.values()) <= set(os.listdir(
        os.path.join(ROOT, "sparse_attention_indexer_head_b200", "csrc")))


def test_input_sets_exceed_twice_l2():
    for step_bytes in (1, 10 ** 6, 28_000_000, 121_071_936, 10 ** 9):
        n = bench.input_sets(step_bytes)
        assert 2 <= n <= 256
        assert n * step_bytes >= 2 * bench.L2_BYTES or n == 256
    assert bench.input_sets(123, requested=3) == 3


def test_peaks_measured_else_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, bench.FALLBACK_TFLOPS, "fallback")
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6552.0, "bf16_tflops": 1500.0}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    assert bench.peaks() == (6552.0, 1500.0, "measured")


def test_replica_throughput_counts_every_rank():
    assert bench.replica_throughput(16, 1, 100, 0.5) == 16 * 100 / 0.5
    assert bench.replica_throughput(16, 8, 100, 0.5) == 8 * 16 * 100 / 0.5
