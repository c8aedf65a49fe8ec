"""Host-side helpers of bench.py (no GPU): the step-traffic figure and the
config both arms print."""
import sys
import types

import bench
import workloads


def test_step_traffic_closed_form():
    # 96 requests at 512K and 50%.  Max pooling: the predict kernel reads D
    # and one V maximum per 32 slots (4.125 B per context slot); the score
    # kernel moves 152 B per kept slot plus one V maximum per 32 kept slots.
    ctx, kept = 96 * 524_292, 25_170_000
    t = bench.step_traffic(ctx, kept, 0.8, 6546.6)
    assert t["bytes_per_step"] == 4.125 * ctx + 152.125 * kept
    assert abs(t["gbs"] - t["bytes_per_step"] / 0.8e-3 / 1e9) < 1e-9
    assert abs(t["frac"] - t["gbs"] / 6546.6) < 1e-12
    # other poolings read V and D whole: 8 B per context slot
    assert bench.step_traffic(ctx, kept, 0.8, 6546.6, "mean")["bytes_per_step"] == 8 * ctx + 152 * kept


def test_both_arms_print_the_same_config():
    args = types.SimpleNamespace(sparsity=0.5, pooling="max")
    wl = workloads.config(2)
    a = bench.headline_config(wl, wl.requests, args, 1)
    b = bench.headline_config(bench.rank_workload(0, 96, 8), 96, args, 1)
    assert a == b
    assert a["workload"] == "serve-96x512K" and a["requests_per_gpu"] == 96
