"""Host-side logic of bench.py (CPU): the measured-traffic figure is reported only
for the kernel sources it was captured from."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write(path, sha, workload="decode_sweep_bf16", value="123456"):
    with open(path, "w") as f:
        f.write("# a capture summary\n")
        f.write("kernel: k\n")
        f.write(f"workload: {workload}\n")
        f.write(f"dram_bytes_per_launch: {value}\n")
        f.write(f"sources_sha256: {sha}\n")


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    f = tmp_path / "traffic.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("decode_sweep_bf16") == (None, "no capture")
    _write(f, bench.kernel_sources_sha256())
    v, src = bench.measured_traffic("decode_sweep_bf16")
    assert v == 123456.0
    _write(f, "0" * 64)  # the kernel changed since the capture
    assert bench.measured_traffic("decode_sweep_bf16") == (None, "kernel changed since the capture")
    _write(f, bench.kernel_sources_sha256(), workload="prefill4096_bf16")
    assert bench.measured_traffic("decode_sweep_bf16")[0] is None
    _write(f, bench.kernel_sources_sha256(), value="not a number")
    assert bench.measured_traffic("decode_sweep_bf16") == (None, "capture file incomplete")


def test_source_hash_covers_the_kernel_files():
    assert all(os.path.exists(p) for p in bench.KERNEL_SOURCES)
    assert any(p.endswith("ffn_gemm.cu") for p in bench.KERNEL_SOURCES)
    assert len(bench.kernel_sources_sha256()) == 64
