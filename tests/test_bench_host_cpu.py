"""Host-side pieces of bench.py that need no GPU: the clock/throttle summary
taken from nvidia-smi's CSV lines, the FLOP count behind MFU, and the
critical-path charge of the profile modes."""
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


def test_critical_path_charges_only_what_extends_the_chain():
    """Kernel records (start, end, name) in start order: a kernel is charged the
    part of it that ends after everything before it, so the charges add up to
    the span from the first start to the last end, a kernel hidden under its
    predecessor costs nothing, and its own duration is kept beside."""
    import bench
    evs = [(0.0, 10.0, "a"), (5.0, 12.0, "b"), (6.0, 11.0, "c"), (13.0, 20.0, "a")]
    agg, tot = bench.critical_path(evs)
    assert tot == 20.0
    assert agg["a"] == [2, 18.0, 17.0]
    assert agg["b"] == [1, 2.0, 7.0]
    assert agg["c"] == [1, 0.0, 5.0]
    assert bench.critical_path([]) == ({}, 0.0)
