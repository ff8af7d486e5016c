"""Host-side contracts of bench.py that need no GPU: the recorded DRAM
traffic is reported only while the kernel sources still hash to the value
recorded with it, and the oracle baseline carries its host description."""

import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _table(tmp_path, rows):
    p = tmp_path / "traffic.md"
    lines = ["| key | sources | sha256 | bytes per launch | note |", "|---|---|---|---|---|"]
    lines += [f"| {k} | {' '.join(src)} | {sha} | {b} | x |" for k, src, sha, b in rows]
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    assert bench.sources_sha256(["kernel.cu"]) == sha
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", _table(tmp_path, [("fa_bwd w", ["kernel.cu"], sha, 123)]))
    assert bench.recorded_traffic("fa_bwd w") == 123.0
    assert bench.recorded_traffic("fa_bwd other") is None          # no row
    src.write_text("// version 2\n")                                 # the kernel changed since
    assert bench.recorded_traffic("fa_bwd w") is None


def test_missing_table_or_source_gives_null(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", str(tmp_path / "absent.md"))
    assert bench.recorded_traffic("fa_bwd w") is None
    monkeypatch.setattr(bench, "TRAFFIC_TABLE", _table(tmp_path, [("fa_bwd w", ["gone.cu"], "0" * 64, 5)]))
    assert bench.recorded_traffic("fa_bwd w") is None


def test_host_info_fields():
    h = bench._host_info(3)
    assert set(h) == {"cpu_model", "logical_cpus", "blas_threads"}
    assert h["blas_threads"] == 3 and h["logical_cpus"] == os.cpu_count()


def test_committed_traffic_rows_parse():
    """Every row of the committed table names sources that exist and a
    64-hex-digit hash; whether it still matches is the bench's business."""
    rows = [r for r in open(bench.TRAFFIC_TABLE).read().splitlines()
            if r.startswith("| ") and not r.startswith("| key") and "|---" not in r]
    assert rows
    for r in rows:
        cells = [c.strip() for c in r.strip().strip("|").split("|")]
        for s in cells[1].split():
            assert os.path.exists(os.path.join(ROOT, s)), s
        assert len(cells[2]) == 64 and int(cells[2], 16) >= 0
        assert float(cells[3]) > 0
