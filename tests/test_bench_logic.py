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


def test_work_accounting():
    # causal pairs: row i of an S x S causal problem sees i + 1 keys; Sq < Sk aligns bottom-right
    assert bench.visible_pairs(4, 4, True) == 10 and bench.visible_pairs(4, 4, False) == 16
    assert bench.visible_pairs(2, 5, True) == 4 + 5
    assert bench.prefill_fwd_flops(1, 2, 4, 4, 8, True) == 4.0 * 8 * 2 * 10
    # decode bytes: K and V once (bf16), Q read and O written (bf16), lse written (fp32)
    assert bench.decode_bytes([3, 5], 4, 2, 8) == 2 * 8 * 2 * 8 * 2 + 2 * 4 * 8 * 2 * 2 + 2 * 4 * 4


def test_reference_arm_counts_its_own_sample():
    # the reference arm's value divides the sample's own FLOPs (one head of the prefill, fwd + 2.5x
    # bwd, and the sampled streams' decode) by its measured seconds
    class P:
        q = type("T", (), {"shape": (1, 16, 4, 8)})()
        k = type("T", (), {"shape": (1, 16, 2, 8)})()
        causal = True

    class Dc:
        meta = {"lengths": [10, 20, 30]}

    f = bench.oracle_sample_flops(P, Dc, 1, 2)
    assert f == pytest.approx(3.5 * bench.prefill_fwd_flops(1, 1, 16, 16, 8, True) + 4.0 * 8 * 4 * 30)
