"""Host-side contracts of bench.py that need no GPU: the recorded DRAM
traffic is reported only while the kernel sources still hash to the value
recorded with it, the roofline peak follows the length of the timed region
and the sampled clock, and the oracle baseline carries its host
description."""

import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _table(tmp_path, rows):
    p = tmp_path / "traffic.json"
    entries = [{"key": k, "sources": list(src), "sha256": sha, "bytes_per_launch": b, "note": "x"}
               for k, src, sha, b in rows]
    p.write_text(json.dumps({"entries": entries}))
    return str(p)


def test_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    assert bench.sources_sha256(["kernel.cu"]) == sha
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _table(tmp_path, [("fa_bwd w", ["kernel.cu"], sha, 123)]))
    assert bench.recorded_traffic("fa_bwd w") == 123.0
    assert bench.recorded_traffic("fa_bwd other") is None          # no entry
    src.write_text("// version 2\n")                                 # the kernel changed since
    assert bench.recorded_traffic("fa_bwd w") is None


def test_missing_table_or_source_gives_null(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.json"))
    assert bench.recorded_traffic("fa_bwd w") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", _table(tmp_path, [("fa_bwd w", ["gone.cu"], "0" * 64, 5)]))
    assert bench.recorded_traffic("fa_bwd w") is None


def test_peak_choice_follows_region_and_clock():
    pk = {"bf16_tflops": 1669.5, "bf16_tflops_sustained": 1411.1}
    # a short region runs at full clock: burst
    assert bench.choose_peak(pk, 41.0, None) == (1669.5, "burst")
    assert bench.choose_peak(pk, 41.0, {"sm_mhz": 1400, "sm_max_mhz": 1965}) == (1669.5, "burst")
    # a long region under the power cap: sustained
    assert bench.choose_peak(pk, 2000.0, {"sm_mhz": 1740, "sm_max_mhz": 1965}) == (1411.1, "sustained")
    assert bench.choose_peak(pk, 2000.0, None) == (1411.1, "sustained")
    # a long region that stayed at the maximum clock: burst
    assert bench.choose_peak(pk, 2000.0, {"sm_mhz": 1965, "sm_max_mhz": 1965}) == (1669.5, "burst")
    # no sustained figure recorded: the burst one
    assert bench.choose_peak({"bf16_tflops": 1500.0}, 5000.0, None)[0] == 1500.0


def test_host_info_fields():
    h = bench._host_info(3)
    assert set(h) == {"cpu_model", "logical_cpus", "blas_threads"}
    assert h["blas_threads"] == 3 and h["logical_cpus"] == os.cpu_count()


def test_committed_traffic_entries_parse():
    """Every committed entry names sources that exist, a 64-hex-digit hash and
    a positive byte count; whether it still matches is the bench's business."""
    entries = json.load(open(bench.TRAFFIC_FILE))["entries"]
    assert entries
    for e in entries:
        for s in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, s)), s
        assert len(e["sha256"]) == 64 and int(e["sha256"], 16) >= 0
        assert float(e["bytes_per_launch"]) > 0
