"""Host-only checks of bench.py's bookkeeping (no GPU): algorithmic bytes
per step, the workloads' call lists, the time-major argument layout, and the
reference arm's JSON line on a bounded sample."""
import json
import subprocess
import sys
import os

import numpy as np

import bench
from segmented_linear_recurrence_b200 import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_per_step():
    # mandatory inputs once + outputs once: GAE 17 B/step (+1 B truncation flag,
    # + trunc_value only where truncated, at 32-byte sectors), 4 B per row bootstrap
    N, T = 64, 256
    d = synthetic.make_inputs("gae", N, T, seed=1, p_term=0.01, p_trunc=0.0)
    assert bench.algorithmic_bytes("gae", d) == 17 * N * T + 4 * N
    d = synthetic.make_inputs("discounted_return", N, T, seed=1, p_term=0.01, p_trunc=0.0)
    assert bench.algorithmic_bytes("discounted_return", d) == 9 * N * T + 4 * N
    d = synthetic.make_affine_inputs(N, T, seed=1)
    assert bench.algorithmic_bytes("affine_scan", d) == 13 * N * T + 4 * N
    # bf16 I/O: r, v, adv, ret 2 B each, the flag 1 B, bootstrap 2 B per row
    d = synthetic.make_inputs("gae", N, T, seed=1, p_term=0.01, p_trunc=0.0)
    assert bench.algorithmic_bytes("gae", d, real_bytes=2) == 9 * N * T + 2 * N


def test_time_major_call_arrays_are_transposes():
    d = synthetic.make_inputs("gae", 5, 7, seed=2, p_term=0.1, p_trunc=0.1)
    rm = bench.call_arrays("gae", d, False)
    tm = bench.call_arrays("gae", d, True)
    for k, a, b in zip(bench.ARG_ORDER["gae"], rm, tm):
        if a is None:
            assert b is None
        elif k in synthetic.PER_ENV_KEYS:
            assert b is a
        else:
            assert b.shape == (7, 5) and b.flags.c_contiguous
            np.testing.assert_array_equal(b, a.T)


def test_workload_calls_cover_estimators_and_windows():
    for wl in ("gae_64x32", "all7_4096x128"):  # the small ones: calls draw their data
        w = synthetic.WORKLOADS[wl]
        calls = bench.workload_calls(wl, 0)
        assert [(e, T) for e, T, _ in calls] == [(e, T) for e in w["estimators"] for T in w["Ts"]]
        # rank shards draw different data
        a = bench.workload_calls(wl, 1)[0][2]
        k = bench.ARG_ORDER[calls[0][0]][0]
        assert not np.array_equal(calls[0][2][k], a[k])
    assert bench.time_major("tm_4096xT") and not bench.time_major(bench.DEFAULT_WORKLOAD)


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "gae_64x32", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         check=True, cwd=ROOT).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
