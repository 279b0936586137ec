"""bench.py's host-side choices, on CPU: the peak that matches the regime of
the timed region, and the fallback figures when no measured peaks exist."""
import bench


PEAKS = {"hbm_gbs": 6540.0, "bf16_tflops": 1632.8, "bf16_tflops_sustained": 1373.9}


def test_short_region_uses_burst_peak():
    peak, src = bench.pick_tensor_peak(PEAKS, "measured", 0.24, {"reasons": ["sw_power_cap"]})
    assert peak == 1632.8 and "burst" in src


def test_long_power_capped_region_uses_sustained_peak():
    peak, src = bench.pick_tensor_peak(PEAKS, "measured", 2.5, {"reasons": ["sw_power_cap"]})
    assert peak == 1373.9 and "sustained" in src


def test_long_region_without_power_cap_uses_burst_peak():
    peak, src = bench.pick_tensor_peak(PEAKS, "measured", 2.5, {"reasons": []})
    assert peak == 1632.8 and "burst" in src


def test_fallback_has_no_sustained_figure():
    fb = dict(bench.FALLBACK_PEAKS)
    assert fb == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
    peak, src = bench.pick_tensor_peak(fb, "fallback", 5.0, {"reasons": ["sw_power_cap"]})
    assert peak == 1590.0 and src.startswith("fallback bf16 burst")
    assert "no sustained figure" in src and "not power-capped" not in src


def test_default_workload_is_the_largest():
    args = bench.parse_args([])
    assert args.config == "175b"
