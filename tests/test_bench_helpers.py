"""Host-side arithmetic of bench.py that needs no GPU."""

import math

import bench


def test_mufu_bound_at_the_video_workload():
    # B1 H12 N32760: one exp2 per (query, key) pair; 148 SMs x 16 exp2/clk at 1965 MHz
    pairs = 1 * 12 * 32760 * 32760
    r = bench.mufu_bound(float(pairs), 6.19, 148, 1965.0)
    assert r["bound"] == "mufu" and r["unit"] == "exp2/s"
    assert math.isclose(r["peak"], 148 * 16 * 1965e6)
    assert math.isclose(r["achieved"], pairs / 6.19e-3)
    assert math.isclose(r["frac"], r["achieved"] / r["peak"])
    # the MUFU floor of this launch: pairs / peak = 2.77 ms
    assert math.isclose(pairs / r["peak"] * 1e3, 2.77, rel_tol=0.01)


def test_job_throughput_counts_every_rank():
    assert math.isclose(bench.job_throughput(6.594e12, 4, 10.0), 4 * 6.594e12 / 1e-2 / 1e12)
