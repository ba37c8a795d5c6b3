"""Host-side arithmetic of bench.py (CPU only): the roofline of each phase, the
error statistics of the bench line, the measured peaks it divides by, and the
step's algorithmic bytes and FLOPs on the headline workload."""
import json
import os
import types

import numpy as np
import pytest
import torch

import bench
import synthetic


def _fake_layer(dt, bytes_, flops):
    return types.SimpleNamespace(PHASES=list(bytes_), dt=dt, phase_bytes=lambda: bytes_,
                                 phase_flops=lambda: flops)


def test_roofline_takes_the_slower_of_bytes_and_flops():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    # fwd: 1 GB at 1000 GB/s = 1 ms against 10 TFLOP at 100 TFLOP/s = 0.1 s -> compute-bound
    # kmap: 2 GB = 2 ms, no flops -> memory-bound
    layer = _fake_layer(torch.bfloat16, {"fwd": 1e9, "kmap": 2e9}, {"fwd": 1e13, "kmap": 0.0})
    rl = bench.roofline_of(layer, {"fwd": 200.0, "kmap": 4.0}, peaks, None)
    assert rl["phases"]["fwd"]["bound"] == "compute"
    assert rl["phases"]["fwd"]["frac"] == pytest.approx(100.0 / 200.0)
    assert rl["phases"]["kmap"]["bound"] == "hbm"
    assert rl["phases"]["kmap"]["frac"] == pytest.approx(2.0 / 4.0)
    assert rl["phases"]["kmap"]["achieved_gbs"] == pytest.approx(500.0)
    assert rl["t_roofline_ms"] == pytest.approx(100.0 + 2.0)


def test_roofline_uses_the_fp32_fma_peak_for_fp32():
    peaks = {"hbm_gbs": 1e6, "bf16_tflops": 1000.0}
    layer = _fake_layer(torch.float32, {"fwd": 1.0}, {"fwd": 72e9})
    rl = bench.roofline_of(layer, {"fwd": 1.0}, peaks, 72.0)  # 72 GFLOP at 72 TFLOP/s = 1 ms
    assert rl["phases"]["fwd"]["bound"] == "compute"
    assert rl["phases"]["fwd"]["frac"] == pytest.approx(1.0)


def test_error_statistics_of_a_known_error():
    ref = np.array([1.0, -2.0, 4.0, 0.0])
    got = ref + np.array([0.01, 0.0, -0.02, 0.0])
    terms = np.array([2.0, 2.0, 4.0, 0.0])  # the last element has no term: left out of the ratios
    st = bench.err_stats(got, ref, terms, torch.bfloat16)
    assert st["max_err_over_max_ref"] == pytest.approx(0.02 / 4.0)
    assert st["pass"] and st["tol"] == 2e-2
    assert st["rel_terms_max"] == pytest.approx(0.005)
    assert st["rel_terms_p50"] == pytest.approx(0.005)
    assert st["elements"] == 4 and st["nonfinite"] == 0
    bad = bench.err_stats(ref + 1.0, ref, terms, torch.float32)
    assert not bad["pass"]


def test_peaks_come_from_the_measured_file():
    peaks = bench.load_peaks()
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        assert peaks["source"] == "measured"
        assert peaks["hbm_gbs"] == pytest.approx(float(d["hbm_gbs"]))
        assert peaks["bf16_tflops"] == pytest.approx(float(d["bf16_tflops"]))
    else:
        assert peaks["source"] == "fallback"


def test_config_names_the_headline_workload_and_its_streams():
    c = bench.config_dict(500_000, 1)
    assert c["workload"].startswith("lidar_train")
    assert c["voxels_per_gpu"] == 500_000 and c["global_batch"] == 4
    assert "second stream" in c["streams"] and "flushed" in c["l2"]
    assert bench.config_dict(500_000, 8)["global_batch"] == 32


def test_headline_step_flops_and_bytes_follow_the_pair_count():
    """FLOPs of the step = 3 passes x 2 P Cin Cout; the forward pass's
    algorithmic bytes on the 500k-voxel workload are the 305.5 MB the
    roofline object divides by (669,006 pairs)."""
    wl = synthetic.WORKLOADS["lidar_train"]
    layer = object.__new__(bench.SubmLayer)  # the arithmetic only: no device buffers
    layer.n, layer.cin, layer.cout, layer.k3, layer.dt = 500_000, wl.cin, wl.cout, 27, torch.bfloat16
    layer.pairs = 669_006
    assert layer.flops() == pytest.approx(3 * 2.0 * 669_006 * 128 * 128)
    pb = layer.phase_bytes()
    assert pb["fwd"] == 305_502_320 and pb["dgrad"] == pb["fwd"]
    assert pb["wgrad"] == 349_652_592
    assert pb["kmap"] == 69_352_048 and pb["hash"] == 16_000_000
