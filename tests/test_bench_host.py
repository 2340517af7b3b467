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
    assert any(p.endswith("ffn_decode.cu") for p in bench.KERNEL_SOURCES)
    assert len(bench.kernel_sources_sha256()) == 64


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the CPU oracle on the host cores) prints one
    JSON line with the contract's keys; it needs no GPU."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3 and d["value"] > 0
    assert d["config"]["workload"] == "decode_sweep_bf16"
    assert d["config"] == bench.workload_config("decode_sweep_bf16", bench.DECODE_BATCHES, 1)  # our arm's config
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
