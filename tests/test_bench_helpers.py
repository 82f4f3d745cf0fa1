"""bench.py's host-side helpers on CPU: the roofline object of the JSON line (tensor
and ALU forms, burst and sustained peaks), the traffic record keyed by the kernel
sources' hash, and the peak-file fallback."""
import hashlib
import os

import pytest

import bench
from matrix_orthogonalising_optimizer_03_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def _prof(ms_apply=0.5, launches=5, flops=6.5e11):
    return {"ns_gram": {"launches": 5, "total_ms": 0.3, "flops": 3.2e11, "bytes": 0.0},
            "ns_apply": {"launches": launches, "total_ms": ms_apply, "flops": flops, "bytes": 0.0},
            "ingest": {"launches": 1, "total_ms": 0.2, "flops": 0.0, "bytes": 1e9}}


def test_roofline_names_the_dominant_tensor_kernel_and_its_fraction():
    w = wl.WORKLOADS["gpt160m"]
    r = bench.roofline(_prof(), w, PEAKS, "measured", "gpt160m", region_ms=90.0)
    assert r["bound"] == "tensor" and r["kernel"] == "ns_apply" and r["unit"] == "TFLOP/s"
    achieved = 6.5e11 / 5 / (0.5e-3 / 5) / 1e12
    assert r["achieved"] == pytest.approx(achieved)
    assert r["peak"] == PEAKS["bf16_tflops"] and r["frac"] == pytest.approx(achieved / 1600.0)
    assert "burst" in r["peak_source"]
    # a timed region of a second or more is compared with the sustained figure
    r2 = bench.roofline(_prof(), w, PEAKS, "measured", "gpt160m", region_ms=1500.0)
    assert r2["peak"] == PEAKS["bf16_tflops_sustained"] and "sustained" in r2["peak_source"]
    # so is a shorter region that ran under the power cap; both fractions are reported
    r3 = bench.roofline(_prof(), w, PEAKS, "measured", "gpt160m", region_ms=900.0,
                        clocks={"reasons": ["sw_power_cap"]})
    assert r3["peak"] == PEAKS["bf16_tflops_sustained"] and "sw_power_cap" in r3["peak_source"]
    assert r3["frac_burst"] == pytest.approx(achieved / 1600.0)
    assert r3["frac_sustained"] == pytest.approx(achieved / 1400.0)
    r4 = bench.roofline(_prof(), w, PEAKS, "measured", "gpt160m", region_ms=900.0,
                        clocks={"reasons": []})
    assert r4["peak"] == PEAKS["bf16_tflops"]


def test_roofline_of_the_fp32_path_is_alu_bound_with_a_fraction():
    w = wl.WORKLOADS["single_128x256"]
    assert w.ns_fp32
    r = bench.roofline(_prof(ms_apply=0.08, flops=3e7), w, PEAKS, "measured", w.name, 20.0)
    assert r["bound"] == "alu" and r["traffic"] is None
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    srcs = ["matrix_orthogonalising_optimizer_03_b200/csrc/ns_tc.cu",
            "matrix_orthogonalising_optimizer_03_b200/csrc/ptx.cuh"]
    h = hashlib.sha256()
    for s in srcs:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    root = tmp_path
    (root / "profiles").mkdir()
    for s in srcs:   # the same sources under a scratch root
        dst = root / s
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, s), "rb").read())
    line = (f"kernel=ns_apply workload=gpt160m bytes_per_launch=123456 sha={h.hexdigest()[:16]} "
            f"sources={','.join(srcs)}\n")
    (root / "profiles" / "traffic.txt").write_text(line)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_record("ns_apply", "gpt160m") == 123456.0
    assert bench.traffic_record("ns_apply", "moe_1b") is None      # other workload
    (root / srcs[1]).write_bytes(b"// changed\n")                   # a kernel source changed
    assert bench.traffic_record("ns_apply", "gpt160m") is None


def test_committed_traffic_record_matches_the_current_sources():
    """The DRAM bytes of the headline's dominant kernel (the 1.5B dense set's ns_apply)
    and of the GPT-160M set's were captured with the tensor-core sources as committed."""
    assert bench.traffic_record("ns_apply", "dense_1p5b") is not None
    assert bench.traffic_record("ns_apply", "gpt160m") is not None


def test_peaks_fall_back_when_the_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
