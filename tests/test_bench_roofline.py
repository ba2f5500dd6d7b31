"""Host logic of the bench line's roofline: the FP8 denominator follows the
run's own clock record (burst peak at the maximum SM clock, sustained peak
under the power cap), every fraction is also given against the problem
statement's ~8 TB/s and ~4.5 PFLOP/s, and the roofline object reproduces by
hand from the breakdown and MEASURED_PEAKS.json."""
import bench


PK = dict(hbm=6457.7, bf16=1662.0, bf16_sus=1404.4, src="measured")


def test_peak_follows_the_clock_record():
    burst, why_b = bench.fp8_peak_for_clock(PK, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert burst == 2 * 1662.0 and "burst" in why_b
    sus, why_s = bench.fp8_peak_for_clock(PK, {"sm_mhz": 1350.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert sus == 2 * 1404.4 and "sustained" in why_s
    none, why_n = bench.fp8_peak_for_clock(PK, None)
    assert none == 2 * 1404.4 and "no clock record" in why_n
    # the clock measured inside the GEMM kernels overrides the sampled median
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped, why_k = bench.fp8_peak_for_clock(PK, at_max, kernel_mhz=1370.0)
    assert capped == 2 * 1404.4 and "inside the GEMM kernels 1370 MHz" in why_k
    full, _ = bench.fp8_peak_for_clock(PK, at_max, kernel_mhz=1960.0)
    assert full == 2 * 1662.0
    kclk = {"pair": {"mhz": 1370.0}, "one_cta": {"mhz": 1450.0}}
    assert bench.gemm_kernel_mhz("wgrad", kclk) == 1370.0 and bench.gemm_kernel_mhz("moe_up", kclk) == 1450.0


def test_roofline_reproduces_from_the_breakdown():
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    # Wgrad at 1460.69 us and quant_x at 37.42 us
    stats = {"wgrad": (1460.69e-6, 1460.69e-6 * 20), "quant_x": (37.42e-6, 37.42e-6 * 20)}
    bd = bench.build_breakdown(stats, PK, 0, {}, clk)
    roof = bench.roofline_for("wgrad", stats, PK, bd, clk)
    flops = 2.0 * 18432 * 7168 * 8192
    achieved = flops / 1460.69e-6 / 1e12
    assert abs(roof["achieved"] - achieved) < 0.1
    assert abs(roof["frac"] - achieved / 3324.0) < 1e-4
    assert abs(roof["frac_spec"] - achieved / 4500.0) < 1e-4
    assert abs(roof["frac_burst"] - achieved / 3324.0) < 1e-4
    # with the in-kernel clock below max the sustained denominator applies
    kclk = {"pair": {"mhz": 1370.0}}
    roof2 = bench.roofline_for("wgrad", stats, PK, bench.build_breakdown(stats, PK, 0, {}, clk, kclk), clk, kclk)
    assert abs(roof2["frac"] - achieved / 2808.8) < 1e-4
    assert abs(bd["wgrad"]["frac_fp8"] - achieved / 3324.0) < 1e-3
    assert bd["wgrad"]["bar_60pct_fp8_spec"] is False
    q = bd["quant_x"]
    gbs = bench.quant_bytes()["quant_x"] / 37.42e-6 / 1e9
    assert abs(q["frac_hbm"] - gbs / 6457.7) < 1e-3 and abs(q["frac_hbm_spec"] - gbs / 8000.0) < 1e-3
    assert q["bar_70pct_hbm_spec"] == (gbs / 8000.0 >= 0.70)
    rq = bench.roofline_for("quant_x", stats, PK, bd, clk)
    assert rq["bound"] == "hbm" and rq["peak"] == 6457.7
