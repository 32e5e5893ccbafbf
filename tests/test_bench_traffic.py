"""bench.py reports the gate_up kernel's captured DRAM traffic only for the kernel source
the capture was taken on: any change to that source makes `roofline.traffic` null until
the counters are taken again.  Host-only (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_traffic_follows_the_captured_kernel_source(tmp_path, monkeypatch):
    import bench
    src = tmp_path / "gemm_swap.cuh"
    with open(bench.GATE_UP_SOURCE, "rb") as f:
        original = f.read()
    src.write_bytes(original)
    monkeypatch.setattr(bench, "GATE_UP_SOURCE", str(src))
    monkeypatch.setattr(bench, "GATE_UP_SOURCE_SHA", bench.kernel_source_sha(str(src)))
    assert bench.gate_up_traffic() == bench.GATE_UP_DRAM_BYTES
    src.write_bytes(original + b"\n// edited\n")          # any edit invalidates the figure
    assert bench.gate_up_traffic() is None
    monkeypatch.setattr(bench, "GATE_UP_SOURCE", str(tmp_path / "missing.cuh"))
    assert bench.gate_up_traffic() is None

