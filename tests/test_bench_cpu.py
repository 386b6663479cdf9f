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
