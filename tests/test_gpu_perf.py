"""Performance regression guard (GPU): a few headline shapes must keep a
floor fraction of the measured copy peak (tests/perf_floor.json).  One
launch's time is taken from CUDA-graph replays of R launches on R input copies
(more than 2x L2 in total, so every launch reads from HBM), after warm-up."""
import json
import os

import numpy as np
import pytest
import torch

import bench
import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build
from segmented_linear_recurrence_b200 import synthetic

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = json.load(open(os.path.join(HERE, "perf_floor.json")))["cases"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_launch_keeps_its_roofline_floor(case):
    est, N, T, A = case["estimator"], case["N"], case["T"], case.get("A", 18)
    tm = bool(case.get("time_major", False))
    d = synthetic.make_inputs(est, N, T, seed=7, p_term=0.02, p_trunc=0.0 if est == "retrace" else 0.005, A=A)
    dev = torch.device("cuda", 0)
    one = bench.DeviceCall(est, T, d, dev, tm)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = int(max(2, min(16, -(-2 * l2 // max(one.bytes, 1)))))
    calls = [one] + [bench.DeviceCall(est, T, d, dev, tm) for _ in range(R - 1)]
    plan = slr.rlscan_query_plan_tm(est, N, T) if tm else slr.rlscan_query_plan(est, N, T, A)
    stream = torch.cuda.Stream(dev)
    slr.rlscan_reserve_workspace(plan["workspace_bytes"], stream)
    with torch.cuda.stream(stream):
        for c in calls:
            c.launch()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c.launch()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = 10
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1000.0 / (reps * R)
    peak, _ = bench.measured_peak()
    frac = one.bytes / (us * 1e3) / peak
    assert slr.rlscan_sync_status() == 0
    assert frac >= case["floor"], f"{case['name']}: {frac:.3f} of measured peak < floor {case['floor']} ({us:.1f} us)"
