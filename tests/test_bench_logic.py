"""Host-side arithmetic of bench.py's roofline object (CPU only, no kernel runs)."""
import pytest

import bench

PEAKS = {"bf16_tflops": 2000.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6000.0}
WORK = {"fwd_sm100": ("tensor", 1.0e11), "bwd_sm100": ("tensor", 2.5e11),
        "bwd_simt_dq": ("alu", None), "decode_split": ("hbm", 5.0e8), "decode_combine": ("hbm", None)}


def entry(prof):
    return bench.roofline_entry(prof, WORK, PEAKS, "measured", traffic_fn=lambda fam, wl: None)


def test_tensor_bound_dominant_kernel():
    # 10 launches of 0.1 ms each: 1e11 FLOPs per 1e-4 s = 1000 TFLOP/s = half the peak
    r = entry({"fwd_sm100": (1.0, 10), "decode_split": (0.5, 10)})
    assert r["kernel"] == "fwd_sm100" and r["bound"] == "tensor"
    assert r["achieved"] == pytest.approx(1000.0)
    assert r["frac"] == pytest.approx(0.5)
    assert r["frac_of_sustained"] == pytest.approx(1000.0 / 1400.0)
    assert r["launch_ms"] == pytest.approx(0.1)


def test_hbm_bound_dominant_kernel():
    # 5e8 bytes per 0.1 ms = 5000 GB/s
    r = entry({"decode_split": (1.0, 10), "fwd_sm100": (0.2, 2)})
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(5000.0)
    assert r["frac"] == pytest.approx(5000.0 / 6000.0)


@pytest.mark.parametrize("dom,bound", [("decode_combine", "hbm"), ("bwd_simt_dq", "alu"), ("mystery", "alu")])
def test_dominant_kernel_without_work_figure_claims_nothing(dom, bound):
    r = entry({dom: (3.0, 2), "fwd_sm100": (1.0, 10)})
    assert r["kernel"] == dom and r["bound"] == bound
    assert r["achieved"] is None and r["frac"] is None and r["peak"] is None


def test_no_profile_no_roofline():
    assert entry({}) is None
