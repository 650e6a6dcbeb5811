"""Host-side pieces of the benchmark that need no GPU: the code hash that keys
the committed DRAM-traffic records, and the summary of clock samples."""

import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402


def test_code_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void k(int* p) {  /* body */\n  p[0] = 1;  // store\n}\n")
    h0 = bench.gemm_code_hash(["k.cu"])
    src.write_text("// a different header\n\n__global__ void k(int* p) {\n  p[0] = 1;   \n}\n/* trailer */\n")
    assert bench.gemm_code_hash(["k.cu"]) == h0
    src.write_text("__global__ void k(int* p) {\n  p[0] = 2;\n}\n")
    assert bench.gemm_code_hash(["k.cu"]) != h0


def test_clock_summary():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.source = "nvml"
    c.samples = [(1800.0, 1965.0, 700.0, {"sw_power_cap"}), (1700.0, 1965.0, 900.0, set()),
                 (1900.0, 1965.0, 800.0, set())]
    s = c.summary()
    assert s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 900.0 and s["power_w_median"] == 800.0
    c.samples = []
    assert c.summary()["samples"] == 0
