"""Host-side pieces of bench.py that need no GPU: the clock/throttle summary
taken from nvidia-smi's CSV lines, and the FLOP count behind MFU."""
import pytest


def test_clock_summary_reasons_and_median():
    import bench
    lines = [
        "1965, 1965, 612.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1785, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1800, 1965, 999.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
    ]
    s = bench.ClockSampler.summarize(lines)
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1800.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_every_slowdown():
    import bench
    lines = ["1200, 1965, 700.0, 0x00000000000000e8, Active, Active, Active, Not Active"]
    s = bench.ClockSampler.summarize(lines)
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_empty():
    import bench
    s = bench.ClockSampler.summarize([])
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == []


def test_flops_per_token_gpt2():
    import bench
    from scratch_decoder_only_b200 import configs as CF
    mc = CF.GPT2_124M.model
    # 6 N + 6 L C (T + 1) with N = 124,475,904 (tied, padded vocabulary)
    assert mc.num_params() == 124_475_904
    assert bench.flops_per_token(mc, 1024) == pytest.approx(6 * 124_475_904 + 6 * 12 * 768 * 1025)
