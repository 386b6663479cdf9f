"""bench.py's CPU legs and host helpers, without a GPU."""
import pytest

import bench


def test_single_thread_oracle_leg_on_the_small_layer():
    r = bench.oracle_single_thread()
    assert r["workload"] == "layer-256x512" and r["cores"] == 1 and r["unit"] == bench.UNIT
    assert r["seconds"] > 0 and r["value"] == pytest.approx(256 * 512 / r["seconds"] / 1e9)


def test_traffic_is_reported_only_for_the_captured_workload_and_sources():
    t = bench.HESSIAN_TRAFFIC
    assert bench.hessian_traffic(t["n"] + 1, t["tokens"]) is None
    assert bench.hessian_traffic(t["n"], t["tokens"] // 2) is None
    # the captured workload: the figure while the kernel's sources are the captured ones, else null
    assert bench.hessian_traffic(t["n"], t["tokens"]) in (None, t["bytes"])


def test_kernel_rooflines_from_a_trace():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "_source": "measured"}
    measured = {"tf32_tflops": 800.0, "fp32_tflops": 70.0}
    trace = {"trailing_update": {"launches": 2, "ms": 1.0, "work": 1e11, "unit": "flop"},
             "sweep": {"launches": 4, "ms": 2.0, "work": 6e9, "unit": "byte"},
             "potrf_inv": {"launches": 32, "ms": 1.0, "work": 7e9, "unit": "flop"},
             "hessian_tc": {"launches": 1, "ms": 1.0, "work": 1.1e12, "unit": "flop"}}
    r = bench.kernel_rooflines(trace, peaks, measured, prepare_ms=2.0, n=4096)
    assert r["trailing_update"]["achieved"] == pytest.approx(300.0)      # 3 passes x 1e11 flop / 1 ms
    assert r["trailing_update"]["frac"] == pytest.approx(300.0 / 800.0)
    assert r["sweep"]["achieved"] == pytest.approx(3000.0) and r["sweep"]["bound"] == "hbm"
    assert r["potrf_inv"]["frac"] == pytest.approx(7.0 / 70.0) and r["potrf_inv"]["bound"] == "alu"
    assert r["hessian_tc"]["frac"] == pytest.approx(1100.0 / 1600.0)
    assert r["prepare (stage)"]["useful_tflops"] == pytest.approx(2 / 3 * 4096 ** 3 / 2e-3 / 1e12)
