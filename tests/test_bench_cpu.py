"""Host-side pieces of bench.py that need no GPU: the algorithmic work models behind the
roofline fields, and the source hash that keeps recorded DRAM traffic attached to its code."""
import os

import bench
from selective_state_space_scan2d_b200 import inputs


def test_forward_model_bounds():
    g = bench.roofline_model(inputs.WORKLOADS["giga"])
    v = bench.roofline_model(inputs.WORKLOADS["vision"])
    assert g["bound"] == "sfu" and v["bound"] == "fp32"
    # per element: x, delta, y plus B and C once per position, shared by the channels
    assert g["bytes_el"] == 3 * 4 + 2 * 16 * 4 / 128
    assert v["bytes_el"] == 3 * 2 + 4 * 2 * 16 * 2 / 192
    assert g["exps_el"] == v["exps_el"] == 16
    assert v["fp32_el"] == 16 * (1 + 4 * 4) + 2


def test_backward_model():
    g = bench.roofline_model_bwd(inputs.WORKLOADS["giga"])
    assert g["bound"] == "fp32"
    assert g["fp32_el"] == 16 * 16 + 4
    assert g["bytes_el"] == 5 * 4 + 2 * 16 * 8 / 128       # x, delta, dy in; dx, ddelta out; B, C in, dB, dC out
    v = bench.roofline_model_bwd(inputs.WORKLOADS["vision"])
    assert v["fp32_el"] == 16 * 16 * 4 + 4


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cuh"
    a.write_text("int f(int x) {\n  return x + 1;  // one more\n}\n")
    b.write_text("/* header */\nconstexpr int k = 3;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ("a.cu", "b.cuh"))
    h0 = bench.kernel_source_hash()
    a.write_text("// a new comment\nint f(int x) {\n\n  return x + 1;\n}\n")
    b.write_text("constexpr int k = 3;  /* same code */\n")
    assert bench.kernel_source_hash() == h0
    a.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.kernel_source_hash() != h0


def test_recorded_traffic_only_for_its_code(monkeypatch):
    """A DRAM-traffic record is reported only while the sources hash to the value recorded
    with it; otherwise the bench reports null."""
    with open(os.path.join(bench.ROOT, "profiles", "scan2d_dram_traffic.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    giga = [r for r in rows if r[0] == "giga:1x128x1024x1024"]
    assert len(giga) == 1
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: giga[0][1])
    assert bench.dram_traffic(inputs.WORKLOADS["giga"]) == float(giga[0][2])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.dram_traffic(inputs.WORKLOADS["giga"]) is None
