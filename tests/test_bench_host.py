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


def test_schedule_summary_in_the_bench_line():
    """config.schedules names each product's planned schedule (host-side
    plan; 148 SMs without a GPU): the 175B-class row products on the
    stream-K tail, the four bf16 row products dynamic, the weight
    gradients static; the 7B-class step static whole tiles throughout."""
    s = bench.plan_summary(2048, 12288, 49152, 8, "bf16")
    assert s == {"F1": "whole tiles, dynamic", "F2": "stream-K tail, dynamic",
                 "B2": "whole tiles, dynamic", "B3": "whole tiles", "B4": "whole tiles",
                 "B5": "stream-K tail, dynamic"}
    assert set(bench.plan_summary(8192, 4096, 16384, 2, "bf16").values()) == {"whole tiles"}
