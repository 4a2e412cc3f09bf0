"""GPU checks of the launch plans and of the bounded look-back wait.

The same inputs go through every block size, the look-back path forced on
where whole rows fit a block, and the scalar (unvectorised) path; each must
match the oracle.  The fault test makes one block withhold its carry (a flag
that nothing sets): its dependants must give up after the configured wait,
report RLSCAN_ERR_TIMEOUT through rlscan_sync_status, and leave the context
usable for the next call.
"""
import numpy as np
import pytest
import torch

import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import synthetic
from segmented_linear_recurrence_b200 import build as slr_build

from .util import check, f32_scalars, gpu_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()


@pytest.fixture
def options():
    yield slr.rlscan_set_option
    for name, default in (("force_lookback", 0), ("force_block", 0), ("force_scalar", 0),
                          ("test_starve_lookback", 0), ("lookback_timeout_ns", 10 ** 9),
                          ("pdl", 1)):
        slr.rlscan_set_option(name, default)


PLAN_CASES = [(4096 // 8, 128), (64, 2048), (5, 5000), (40, 96), (33, 1001), (7, 3)]


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
@pytest.mark.parametrize("block", [128, 192, 256, 320, 384, 448, 512])
@pytest.mark.parametrize("lookback", [0, 1])
def test_every_plan_matches_oracle(est, block, lookback, options):
    if est == "retrace" and block not in (128, 256):
        pytest.skip("Retrace stages its action rows with 128- or 256-thread blocks")
    options("force_block", block)
    options("force_lookback", lookback)
    for N, T in PLAN_CASES:
        d = synthetic.make_inputs(est, N, T, seed=900 + N + T, p_term=0.01, p_trunc=0.01, A=6,
                                  with_init=True)
        plan = slr.rlscan_query_plan(est, N, T, 6)
        assert plan["block_threads"] == block
        if lookback:
            assert plan["lookback"] == 1
        check(est, d, synthetic.SCALARS[est], what=f"block={block} lookback={lookback} N={N} T={T}")


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_scalar_path_matches_vector_path(est, options):
    d = synthetic.make_inputs(est, 48, 1536, seed=71, p_term=0.01, p_trunc=0.01, A=6,
                              with_init=True)
    s = f32_scalars(est, synthetic.SCALARS[est])
    vec = gpu_run(est, d, **s)
    options("force_scalar", 1)
    sca = gpu_run(est, d, **s)
    for a, b in zip(vec, sca):
        if a is not None:
            np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_plain_launch_matches_programmatic_launch(est, options):
    # back-to-back calls with and without programmatic dependent launch
    d = synthetic.make_inputs(est, 96, 700, seed=70, p_term=0.01, p_trunc=0.01, A=6,
                              with_init=True)
    s = f32_scalars(est, synthetic.SCALARS[est])
    pdl = [gpu_run(est, d, **s) for _ in range(3)]
    options("pdl", 0)
    plain = gpu_run(est, d, **s)
    for run in pdl:
        for a, b in zip(run, plain):
            if a is not None:
                np.testing.assert_array_equal(a, b)


def test_lookback_survives_many_calls_on_one_stream(options):
    # the per-stream workspace is reused: tickets wrap and the epoch advances
    d = synthetic.make_inputs("td_lambda", 8, 30_000, seed=72, p_term=0.0005)
    s = f32_scalars("td_lambda", synthetic.SCALARS["td_lambda"])
    first = gpu_run("td_lambda", d, **s)
    for _ in range(20):
        np.testing.assert_array_equal(first[0], gpu_run("td_lambda", d, **s)[0])
    d2 = synthetic.make_inputs("td_lambda", 3, 70_001, seed=73, p_term=0.0005)
    check("td_lambda", d2, synthetic.SCALARS["td_lambda"], what="grown workspace")
    assert slr.rlscan_sync_status() == 0


def test_lookback_on_two_streams(options):
    d = synthetic.make_inputs("gae", 4, 50_000, seed=74, p_term=0.0005, p_trunc=0.0005)
    s = f32_scalars("gae", synthetic.SCALARS["gae"])
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        a = gpu_run("gae", d, stream=s1, **s)
    with torch.cuda.stream(s2):
        b = gpu_run("gae", d, stream=s2, **s)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_withheld_carry_times_out_and_reports(options):
    # Two rows of 40_000 steps: 10 chunks per row with 1024-step chunks.  The
    # block holding the first ticket (the last chunk of the last row) never
    # publishes; the chunk before it waits 20 ms, gives up and reports.
    options("lookback_timeout_ns", 20_000_000)
    options("force_block", 256)
    options("test_starve_lookback", 1)
    d = synthetic.make_inputs("discounted_return", 2, 40_000, seed=75, p_term=0.0)
    d["terminated"][:] = 0
    s = f32_scalars("discounted_return", synthetic.SCALARS["discounted_return"])
    assert slr.rlscan_sync_status() == 0
    gpu_run("discounted_return", d, **s)
    assert slr.rlscan_sync_status() == 4  # RLSCAN_ERR_TIMEOUT
    # the context stays usable and the next call is correct
    options("test_starve_lookback", 0)
    check("discounted_return", d, synthetic.SCALARS["discounted_return"], what="after timeout")
    assert slr.rlscan_sync_status() == 0


@pytest.mark.parametrize("est,N,T", [("gae", 8, 20_000), ("vtrace", 512, 128), ("elig_trace", 4, 9_999)])
def test_graph_capture_and_replay(est, N, T):
    # Tickets wrap and the look-back epoch advances on the device, so a call
    # captured once can be replayed any number of times.
    d = synthetic.make_inputs(est, N, T, seed=76, p_term=0.001, p_trunc=0.001, with_init=True)
    s = f32_scalars(est, synthetic.SCALARS[est])
    from .util import OUTPUT_NAMES, assert_parity, oracle_run, to_dev
    t = to_dev(d)
    cap = torch.cuda.Stream()
    plan = slr.rlscan_query_plan(est, N, T)
    slr.rlscan_reserve_workspace(plan["workspace_bytes"], cap)
    fn = getattr(slr, f"rlscan_{est}")
    order = {"gae": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
             "vtrace": ("log_rhos", "rewards", "values", "bootstrap", "terminated", "truncated",
                        "trunc_value"),
             "elig_trace": ("inputs", "init_trace", "terminated", "truncated")}[est]
    outs = {k: torch.empty(N, T, device="cuda") for k in OUTPUT_NAMES[est]}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        fn(*[t.get(k) for k in order], **s, **outs)
    ref = oracle_run(est, d, **s)
    for _ in range(5):
        for o in outs.values():
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert_parity(est, tuple(outs[k].cpu().numpy() for k in OUTPUT_NAMES[est]), ref, what="replay")
    assert slr.rlscan_sync_status() == 0


# Look-back with rows of whole chunks (T a multiple of the chunk): tickets
# interleave the rows (every row's first chunk in dependency order, then every
# row's second, ...).  Mixed with a T whose chunks straddle rows (flat order)
# for the 16-step estimators.
@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_row_interleaved_tickets_match_oracle(est):
    cases = {"retrace": [(37, 4096), (9, 8192)], "elig_trace": [(37, 16384), (130, 12288), (3, 10000)],
             "episodic_prefix_sum": [(37, 16384), (130, 12288), (3, 10000)]}.get(
                 est, [(37, 16384), (130, 8192), (3, 6144)])
    for N, T in cases:
        d = synthetic.make_inputs(est, N, T, seed=990 + N + T, p_term=0.002, p_trunc=0.002, A=6,
                                  with_init=True)
        assert slr.rlscan_query_plan(est, N, T, 6)["lookback"] == 1
        check(est, d, synthetic.SCALARS[est], what=f"interleaved N={N} T={T}")
