"""The bench's arithmetic on the host: peak choice from the clock record,
the whole-step roofline side, the per-layer figures, the traffic lookup and
its source label."""

import pytest

import bench
import workloads as WL

PEAKS = {"hbm_gbs": 6550.0, "bf16_tflops": 1670.0, "bf16_tflops_sustained": 1385.0}


def test_clocks_capped_only_when_the_clock_really_fell():
    assert not bench.clocks_capped({})
    assert not bench.clocks_capped({"sm_mhz": None, "sm_max_mhz": 1965})
    # touching the power cap at full clocks counts as full clocks
    assert not bench.clocks_capped({"sm_mhz": 1961, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    assert not bench.clocks_capped({"sm_mhz": 0.9 * 1965, "sm_max_mhz": 1965, "reasons": []})
    # a power-capped loop sampled inside its timed region
    assert bench.clocks_capped({"sm_mhz": 1492, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    assert bench.clocks_capped({"sm_mhz": 1300, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})


def test_tensor_peak_follows_the_clocks():
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    low = {"sm_mhz": 1300, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    assert bench.tensor_peak(PEAKS, "measured", full) == (1670.0, "measured bf16 dense (burst)")
    peak, src = bench.tensor_peak(PEAKS, "measured", low)
    assert peak == 1385.0 and "sustained" in src


def test_step_roofline_sides():
    clk = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    llama = WL.WORKLOADS["llama"]
    r = bench.step_roofline(llama, 4.0, clk, PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(llama.gemm_flops() / 4e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1670.0)
    decode = WL.WORKLOADS["decode"]
    r = bench.step_roofline(decode, 0.24, clk, PEAKS, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(bench.block_bytes(decode) / 0.24e-3 / 1e9)
    assert r["intensity_flop_per_byte"] < r["ridge_flop_per_byte"]


def test_layer_figures_add_up():
    w = WL.WORKLOADS["wide"]
    kernels = {"column": 0.35, "row": 0.38, "reduce": 0.053, "sum": 0.783}
    clk = {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": []}
    f = bench.layer_figures(w, kernels, clk, PEAKS, "measured")
    assert f["column"]["TFLOP/s"] == pytest.approx(bench.column_flops(w) / 0.35e-3 / 1e12)
    assert f["row"]["TFLOP/s"] == pytest.approx(bench.row_flops(w) / 0.38e-3 / 1e12)
    assert f["reduce"]["bytes"] == (w.p + 1) * w.T * w.d * 4
    assert f["reduce"]["GB/s"] == pytest.approx(f["reduce"]["bytes"] / 0.053e-3 / 1e9)
    assert f["column"]["ms_x_mhz"] == pytest.approx(0.35 * 1900)
    assert f["step_ms"] == 0.783 and f["peak"]["bf16_tflops"] == 1670.0
    toy = WL.WORKLOADS["toy"]   # fp32: no bf16 fraction
    f = bench.layer_figures(toy, kernels, clk, PEAKS, "measured")
    assert f["column"]["frac_bf16_peak"] is None


def test_traffic_entry_labels_its_source():
    e = bench.traffic_entry("llama/column")
    if e["traffic"] is None:        # table entry taken on other kernel code
        assert e["traffic_source"].startswith("none")
    else:
        assert e["traffic"] > 0 and "profiles/ncu_traffic.json[llama/column]" in e["traffic_source"]
    e = bench.traffic_entry("no/such")
    assert e["traffic"] is None and "no ncu figure" in e["traffic_source"]


def test_whole_job_value_and_tokens_override():
    assert bench.whole_job_value(2e12, 4, 10.0) == pytest.approx(8e14)
    import dataclasses
    w = dataclasses.replace(WL.WORKLOADS["llama"], T=1024, name="llama_T1024")
    assert w.gemm_flops() * 4 == WL.WORKLOADS["llama"].gemm_flops()


def test_clock_samples_are_taken_from_the_timed_region():
    """ClockSampler keeps the nvidia-smi samples whose timestamps fall inside
    the timed region: an idle sample before it (low clock, no load) and a
    throttled one after it do not count; the loaded samples' median does."""
    import datetime
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5).timestamp()

    def line(dt, mhz, watts, power_cap="Not Active", thermal="Not Active"):
        ts = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return (f"{ts}, 0, {mhz}, 1965, {watts}, 0x0, Not Active, Not Active, {thermal}, "
                f"{power_cap}\n")

    lines = [line(-0.2, 345, 90.0),                       # idle, before the region
             line(0.01, 1965, 900.0), line(0.03, 1950, 950.0, power_cap="Active"),
             line(0.05, 1965, 910.0), line(0.07, 120, 100.0),   # a dip in load inside
             line(0.5, 1200, 950.0, thermal="Active")]    # after the region
    rows = bench.ClockSampler.parse(lines)
    assert len(rows) == 6
    s = bench.ClockSampler.summarise(rows, t0, t0 + 0.08)
    assert s["samples"] == 4 and s["window"] == "timed region"
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    # no sample inside the window: all samples, said so
    s = bench.ClockSampler.summarise(rows, t0 + 10, t0 + 11)
    assert s["samples"] == 6 and s["window"].startswith("whole sampling")
    assert "sw_thermal_slowdown" in s["reasons"]
    assert bench.ClockSampler.summarise([], t0, t0 + 1)["reasons"] == ["no samples"]
