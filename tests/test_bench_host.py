"""bench.py's host-side helpers: the roofline's DRAM-traffic lookup (profiles/ncu_dram_traffic.txt
keyed by a digest of the kernel sources) and the choice of the tensor peak by the clock."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_source_digest_covers_kernel_and_tile_schedule(tmp_path, monkeypatch):
    d0 = bench.source_digest("gemm_gate_up")
    assert len(d0) == 16 and d0 == bench.source_digest("gemm_down")  # same sources
    assert bench.source_digest("router") != d0
    # a change to the tile schedule changes the digest
    csrc = tmp_path / "mixture_experts_layer_score_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("gemm_sm100.cu", "grouped_tiles.cuh"):
        (csrc / name).write_bytes(open(os.path.join(ROOT, bench.CSRC, name), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.source_digest("gemm_gate_up") == d0
    (csrc / "grouped_tiles.cuh").write_bytes(b"// changed\n" + (csrc / "grouped_tiles.cuh").read_bytes())
    assert bench.source_digest("gemm_gate_up") != d0


def test_captured_traffic_prefers_the_benchmarked_workload(tmp_path, monkeypatch):
    digest = bench.source_digest("gemm_gate_up")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_dram_traffic.txt").write_text(
        "# comment line\n"
        f"gemm_gate_up {digest} 300 100 small_case kernel\n"
        f"gemm_gate_up {digest} 220 200 big_case kernel\n"
        "gemm_gate_up 0000000000000000 999 1 big_case stale\n")
    csrc = tmp_path / "mixture_experts_layer_score_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("gemm_sm100.cu", "grouped_tiles.cuh", "gemm_gateup_pair_sm100.cu"):
        (csrc / name).write_bytes(open(os.path.join(ROOT, bench.CSRC, name), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert abs(bench.captured_traffic("gemm_gate_up", 400.0, "single", "big_case") - 440.0) < 1e-9  # 220/200
    assert abs(bench.captured_traffic("gemm_gate_up", 400.0, "single", "other") - 1200.0) < 1e-9    # first line
    assert bench.captured_traffic("gemm_down", 400.0, "single", "big_case") is None       # no capture
    assert bench.captured_traffic("gemm_gate_up", 400.0, "pair", "big_case") is None      # other kernel sources


def test_tensor_peak_follows_the_clock():
    assert bench.tensor_peak_key({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}) == "bf16_tflops"
    assert bench.tensor_peak_key({"sm_mhz": 1320.0, "sm_max_mhz": 1965.0}) == "bf16_tflops_sustained"
