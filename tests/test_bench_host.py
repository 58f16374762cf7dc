"""Host-side logic of bench.py (no GPU): the ncu traffic record is used only
for the kernel source it was captured from, and the reference arm (the CPU
oracle timed on the decode step) prints one JSON line with the contract's keys."""
import contextlib
import hashlib
import io
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_tree(tmp_path, source: bytes, recorded: bytes):
    csrc = tmp_path / "block_scaled_w8a8_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemm_decode.cu").write_bytes(source)
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"source_file": "gemm_decode.cu",
           "source_sha256": hashlib.sha256(recorded).hexdigest(),
           "dram_bytes_per_launch": 16.9e6, "capture": "ncu ..."}
    (prof / "roofline_traffic.json").write_text(json.dumps(rec))


def test_traffic_record_used_for_the_captured_kernel(tmp_path, monkeypatch):
    _fake_tree(tmp_path, b"kernel v1", b"kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    val, src = bench.load_traffic("gemm_decode.cu")
    assert val == pytest.approx(16.9e6) and src == "ncu ..."


def test_traffic_is_null_once_the_kernel_changed(tmp_path, monkeypatch):
    _fake_tree(tmp_path, b"kernel v2", b"kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    val, why = bench.load_traffic("gemm_decode.cu")
    assert val is None and "changed" in why


def test_traffic_is_null_without_a_record(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("gemm_decode.cu")[0] is None


def test_reference_arm_prints_the_contract_line(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(bench.argparse.Namespace(gpus=1, steps=1, warmup=0))
    assert rc == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
