"""Host-side arithmetic of bench.py that the JSON line depends on: the
algorithmic byte and FLOP counts of the workloads, and the rule that a
captured DRAM traffic figure is reported only while the kernel sources still
hash to the value recorded with it.  CPU only."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_algorithmic_bytes_of_the_decode_layer():
    # NF4: codes K/2 + fp32 absmax K/64*4 per weight row, x read once, out written
    gu = bench.gemv_bytes("nf4", 8, 1536, 2048, 1)
    assert gu == 8 * 1536 * (2048 // 2 + 2048 // 64 * 4) + 1 * 2048 * 2 + 8 * 1536 * 2
    assert gu == 14_184_448
    assert bench.gemv_bytes("nf4", 8, 2048, 768, 8) == 7_122_944
    # MXFP4: codes K/2 + one e8m0 byte per 32
    assert bench.gemv_bytes("mxfp4", 4, 5760, 2880, 1) == 35_303_040
    assert bench.gemv_bytes("mxfp4", 4, 2880, 2880, 4) == 17_671_680


def test_algorithmic_flops():
    assert bench.gemm_flops(32768, 1536, 2048) == 2 * 32768 * 1536 * 2048
    assert abs(bench.gemm_flops(8192, 5760, 2880) / 1e9 - 271.79) < 0.01


def _with_traffic(tmp_path, monkeypatch, entry):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({"k": entry}))
    src = tmp_path / "src.cu"
    src.write_text("kernel source v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return src


def test_traffic_reported_only_while_the_source_hash_matches(tmp_path, monkeypatch):
    digest = hashlib.sha256(b"kernel source v1\n").hexdigest()
    src = _with_traffic(tmp_path, monkeypatch,
                        {"bytes": 123, "sources": ["src.cu"], "source_sha256": digest})
    assert bench.load_traffic("k") == 123
    src.write_text("kernel source v2\n")          # the kernel changed since the capture
    assert bench.load_traffic("k") is None
    assert bench.load_traffic("missing") is None
