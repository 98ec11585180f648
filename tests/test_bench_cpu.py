"""The benchmark's bookkeeping, on the CPU: the algorithmic bytes its roofline
divides by, the rule that a committed DRAM-traffic record is used only while
the kernel sources are the ones it was measured on, and the peak it reads."""
import json
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("sum_M,K,E", [(80768, 7168, 256), (768, 512, 4), (128, 128, 1)])
def test_algorithmic_bytes(sum_M, K, E):
    """amax reads x (2 B/elem) and writes both amax vectors; the cast reads x
    and both vectors and writes codes (1/2 B) and E4M3 scales (1/16 B) per
    element and direction plus both decode-scale vectors: 5.125 B/elem in all."""
    N = sum_M * K
    b = bench.algorithmic_bytes(sum_M, K, E)
    assert b["amax"] == 2 * N + 4 * sum_M + 4 * E * K
    assert b["cast"] == 2 * N + 2 * (N // 2 + N // 16) + 8 * sum_M + 8 * E * K
    assert b["step"] == b["amax"] + b["cast"]
    assert b["step"] == 5.125 * N + 12 * sum_M + 12 * E * K
    assert bench.output_bytes(sum_M, K, E) == N + N // 8 + 4 * sum_M + 4 * E * K


def _fake_root(tmp_path, record):
    """A copy of the kernel sources and a traffic record under tmp_path."""
    src = os.path.join(ROOT, "nvfp4_row_scaled_b200", "csrc")
    shutil.copytree(src, tmp_path / "nvfp4_row_scaled_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(record))


def test_kernel_source_lists_exist():
    d = os.path.join(ROOT, "nvfp4_row_scaled_b200", "csrc")
    for files in bench.KERNEL_SOURCES.values():
        for f in files:
            assert os.path.exists(os.path.join(d, f)), f


def test_traffic_record_only_for_the_sources_it_was_measured_on(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _fake_root(tmp_path, {})
    h = bench.kernel_source_hash("group_cast_plain_kernel")
    rec = {"group_cast_plain_kernel": {"workload": "w", "source_hash": h, "bytes_per_launch": 123}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_record("group_cast_plain_kernel", "w") == 123
    assert bench.traffic_record("group_cast_plain_kernel", "other workload") is None
    assert bench.traffic_record("group_amax_kernel", "w") is None
    # a change to a source of another kernel only keeps the record
    f = tmp_path / "nvfp4_row_scaled_b200" / "csrc" / "mx_cast.cuh"
    f.write_text(f.read_text() + "\n")
    assert bench.traffic_record("group_cast_plain_kernel", "w") == 123
    # any change to one of the kernel's own sources retires it
    f = tmp_path / "nvfp4_row_scaled_b200" / "csrc" / "codec.cuh"
    f.write_text(f.read_text() + "\n")
    assert bench.kernel_source_hash("group_cast_plain_kernel") != h
    assert bench.traffic_record("group_cast_plain_kernel", "w") is None


def test_peak_from_measured_file_else_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6400.5}))
    assert bench.hbm_peak() == (6400.5, "measured")
