"""Host logic of bench.py's roofline: the dominant kernel, its companion launches and the
L2 bound (CPU only)."""
import os
import sys
import types

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0, "source": "test",
         "l2_gather_gbs": 16000.0}


def _wl(spec, name="w"):
    return types.SimpleNamespace(roofline_spec=lambda: dict(spec), name=name)


def _prof(**ms):
    return {k: {"total_ms": v, "timed_launches": 10, "launches": 10} for k, v in ms.items()}


def test_companion_time_counts_with_the_top_kernel():
    spec = {"ring": [("hbm", 0.281, "GB/s"), ("tensor", 0.0687, "TFLOP/s")], "_with": {"ring": ["tc"]}}
    out, stages = bench.roofline(_wl(spec), _prof(ring=2.70, tc=0.07, other=0.5), PEAKS)
    assert out["kernel"] == "ring" and out["includes"] == ["tc"]
    assert out["per_launch_ms"] == pytest.approx(0.277)
    # 0.281 GB per launch over 0.277 ms; the byte roofline binds (0.281/6000 > 0.0687/1500)
    assert out["bound"] == "hbm"
    assert out["achieved"] == pytest.approx(0.281 / 0.277e-3, rel=1e-3)
    assert out["frac"] == pytest.approx(0.281 / 0.277e-3 / 6000.0, rel=1e-3)
    assert out["secondary"]["bound"] == "tensor"
    assert stages["tc"] == pytest.approx(0.007)


def test_l2_bound_uses_the_measured_gather_ceiling():
    spec = {"sparse_attn": [("l2", 33.3, "GB/s"), ("tensor", 0.18, "TFLOP/s")]}
    out, _ = bench.roofline(_wl(spec), _prof(sparse_attn=45.2), PEAKS)
    assert out["bound"] == "l2" and out["peak"] == 16000.0
    assert out["frac"] == pytest.approx(33.3 / 4.52e-3 / 16000.0, rel=1e-3)


def test_a_kernel_without_a_spec_reports_no_roofline():
    out, _ = bench.roofline(_wl({"a": [("hbm", 1.0, "GB/s")]}), _prof(b=1.0), PEAKS)
    assert out["kernel"] == "b" and out["frac"] is None
