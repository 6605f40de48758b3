"""Host-side logic of bench.py that needs no GPU: which measured GEMM peak a
forward timing is compared with, and which clock samples describe the timed
region."""
import bench

PEAKS = {"hbm_gbs": 6537.3, "bf16_tflops": 1647.8, "bf16_tflops_sustained": 1379.4,
         "sm_max_mhz": 1965.0, "sustained_sm_mhz": 1252.0, "source": "measured"}


def test_region_without_power_cap_takes_the_burst_peak():
    clocks = {"sm_mhz": 1965.0, "reasons": []}
    regime, peak, why = bench.tensor_peak_regime(PEAKS, clocks, 87.0)
    assert regime == "burst" and peak == 1647.8 and "not active" in why
    # 1250 TF/s in that regime is 0.76 of the measured burst GEMM
    assert abs(1250.0 / peak - 0.7586) < 1e-3


def test_power_capped_region_takes_the_sustained_peak():
    # the forward pass at the cap keeps a higher clock than a GEMM at the cap:
    # the cap, not the clock, names the regime
    clocks = {"sm_mhz": 1661.0, "reasons": ["sw_power_cap"]}
    regime, peak, _ = bench.tensor_peak_regime(PEAKS, clocks, 945.0)
    assert regime == "sustained" and peak == 1379.4


def test_without_reasons_the_clock_decides_and_without_clocks_the_length():
    assert bench.tensor_peak_regime(PEAKS, {"sm_mhz": 1609.0}, 900.0)[0] == "burst"
    assert bench.tensor_peak_regime(PEAKS, {"sm_mhz": 1600.0}, 900.0)[0] == "sustained"
    assert bench.tensor_peak_regime(PEAKS, {"sm_mhz": None}, 500.0)[0] == "burst"
    assert bench.tensor_peak_regime(PEAKS, {}, 4000.0)[0] == "sustained"


def _line(sm, reason_cap="Not Active"):
    return (f"0, {sm}, 1965, 900.5, 0x0000000000000004, Not Active, Not Active, Not Active, "
            f"{reason_cap}\n")


def test_clock_summary_keeps_the_samples_inside_the_timed_region():
    stamped = [(0.0, _line(1965)), (0.1, _line(1965)), (1.0, _line(1500, "Active")),
               (1.1, _line(1550, "Active")), (1.2, _line(1600)), (2.0, _line(1965))]
    c = bench.ClockSampler.parse(stamped, 0.95, 1.25)
    assert c["samples_in_timed_region"] == 3 and c["sm_mhz"] == 1550.0
    assert c["reasons"] == ["sw_power_cap"] and c["window"] == "timed region"
    # no sample inside a very short region: all samples are summarised, and said so
    c = bench.ClockSampler.parse(stamped, 0.5, 0.6)
    assert c["samples_in_timed_region"] == 0 and c["samples"] == 6
    assert c["window"].startswith("around")
    # malformed lines are skipped
    assert bench.ClockSampler.parse([(0.0, "garbage\n")], 0, 1)["sm_mhz"] is None
