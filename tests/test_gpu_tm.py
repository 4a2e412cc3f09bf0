"""GPU parity of the time-major entry points (rlscan_*_tm): every per-step
array [T, N], element (t, n) at t * N + n.  The oracle is the row-major
oracle on the transposed arrays (the recurrences run along T per environment
whatever the storage order); the generic affine scan is also checked against
the oracle's own time-major loop.  Same bar as the row-major calls:
|gpu - ref| <= 1e-4 (1 + |ref|) element by element, int32 bit-exact, on short
windows (one chunk, several environments per block), look-back chains along
T, ragged N and T, host tensors, graph replay and a withheld carry."""
import numpy as np
import pytest
import torch

import oracle
import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build
from segmented_linear_recurrence_b200 import synthetic

from .util import TOL, assert_parity, f32_scalars, oracle_run

pytestmark = pytest.mark.gpu

TM_ESTIMATORS = ("gae", "vtrace", "td_lambda", "discounted_return", "elig_trace", "episodic_prefix_sum")
PER_ENV = ("bootstrap", "init_trace", "init")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()


@pytest.fixture
def options():
    yield slr.rlscan_set_option
    for name, default in (("force_lookback", 0), ("test_starve_lookback", 0), ("lookback_timeout_ns", 10**9)):
        slr.rlscan_set_option(name, default)


def transpose(d):
    """Row-major [N, T] arrays to time-major [T, N]; [N] arrays unchanged."""
    return {k: (None if v is None else (v if k in PER_ENV else np.ascontiguousarray(v.T))) for k, v in d.items()}


def tm_run(est, dt, device="cuda", stream=None, **scal):
    """One time-major call on the arrays of `dt` ([T, N]); numpy outputs [T, N]."""
    t = {k: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in dt.items()}
    if est == "gae":
        res = slr.rlscan_gae_tm(t["rewards"], t["values"], t["bootstrap"], t["terminated"], t.get("truncated"),
                                t.get("trunc_value"), stream=stream, **scal)
    elif est == "vtrace":
        res = slr.rlscan_vtrace_tm(t["log_rhos"], t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                                   t.get("truncated"), t.get("trunc_value"), stream=stream, **scal)
    elif est == "td_lambda":
        res = slr.rlscan_td_lambda_tm(t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                                      t.get("truncated"), t.get("trunc_value"), stream=stream, **scal)
    elif est == "discounted_return":
        res = slr.rlscan_discounted_return_tm(t["rewards"], t.get("bootstrap"), t["terminated"], t.get("truncated"),
                                              t.get("trunc_value"), stream=stream, **scal)
    elif est == "elig_trace":
        res = slr.rlscan_elig_trace_tm(t["inputs"], t.get("init_trace"), t["terminated"], t.get("truncated"),
                                       stream=stream, **scal)
    elif est == "episodic_prefix_sum":
        res = slr.rlscan_episodic_prefix_sum_tm(t["x"], t["terminated"], t.get("truncated"), stream=stream)
    elif est == "affine_scan":
        res = slr.rlscan_affine_scan_tm(t["a"], t["b"], t.get("reset"), t.get("init"),
                                        reverse=bool(scal.get("reverse", False)), stream=stream)
    else:
        raise ValueError(est)
    res = res if isinstance(res, tuple) else (res,)
    return tuple(None if r is None else r.cpu().numpy() for r in res)


def inputs(est, N, T, seed):
    if est == "affine_scan":
        return synthetic.make_affine_inputs(N, T, seed=seed, p_reset=0.01)
    return synthetic.make_inputs(est, N, T, seed=seed, p_term=0.01, p_trunc=0.01, with_init=True)


def check_tm(est, N, T, seed, scal=None, what=""):
    d = inputs(est, N, T, seed)
    s = f32_scalars(est, dict(synthetic.SCALARS.get(est, {}) if scal is None else scal))
    got = tm_run(est, transpose(d), **s)
    ref = oracle_run(est, d, **s)
    assert_parity(est, tuple(None if g is None else np.ascontiguousarray(g.T) for g in got), ref,
                  what=f"time-major N={N} T={T} {what}")
    return got


# Shapes: one chunk with 1, 2, 4 and 8 time slices per block (T <= 8, 16, 32,
# 64), look-back chains (T > 64), ragged environments (N not a multiple of
# 32) and windows (T not a multiple of 8), and the configs' row shapes.
CASES = [(4096, 512), (64, 2048), (33, 1001), (1000, 64), (300, 32), (130, 7), (257, 129), (5, 5000),
         (96, 16), (2, 40_001), (4096, 128)]


@pytest.mark.parametrize("est", TM_ESTIMATORS + ("affine_scan",))
@pytest.mark.parametrize("N,T", CASES)
def test_time_major_matches_oracle(est, N, T):
    check_tm(est, N, T, seed=3000 + N + T)


@pytest.mark.parametrize("est", TM_ESTIMATORS + ("affine_scan",))
def test_time_major_forced_lookback(est, options):
    # Shorter chunks: carries chain even where one block would cover T.
    options("force_lookback", 1)
    for N, T in [(300, 32), (96, 16), (40, 63), (70, 9)]:
        check_tm(est, N, T, seed=3100 + N + T, what="forced look-back")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("N,T", [(64, 2048), (33, 1001), (300, 32), (2, 40_001)])
def test_affine_time_major_matches_time_major_oracle(N, T, reverse):
    d = synthetic.make_affine_inputs(N, T, seed=3200 + N + T, p_reset=0.01, a_low=-1.0, a_high=1.0)
    dt = transpose(d)
    got = tm_run("affine_scan", dt, reverse=reverse)[0].astype(np.float64)
    ref = oracle.affine_scan_tm(dt["a"], dt["b"], dt["reset"], dt["init"], reverse=reverse)
    err = np.abs(got - ref)
    assert (err <= TOL * (1.0 + np.abs(ref))).all(), float((err / (1.0 + np.abs(ref))).max())


@pytest.mark.parametrize("est", TM_ESTIMATORS)
def test_time_major_equals_row_major_on_device(est):
    # Same inputs through both layouts: the same recurrence, so the outputs
    # agree to fp32 reassociation.
    import tests.util as U
    d = inputs(est, 200, 777, seed=3300)
    s = f32_scalars(est, synthetic.SCALARS[est])
    rm = U.gpu_run(est, d, **s)
    tm = tm_run(est, transpose(d), **s)
    assert_parity(est, tuple(None if g is None else np.ascontiguousarray(g.T) for g in tm),
                  tuple(None if g is None else g.astype(np.float64) for g in rm), what="tm vs rm")


def test_time_major_host_tensors():
    d = inputs("gae", 50, 300, seed=3400)
    s = f32_scalars("gae", synthetic.SCALARS["gae"])
    got = tm_run("gae", transpose(d), device="cpu", **s)
    ref = oracle_run("gae", d, **s)
    assert_parity("gae", tuple(np.ascontiguousarray(g.T) for g in got), ref, what="host tensors")


@pytest.mark.parametrize("N", [37, 64])
def test_time_major_unaligned_views(N):
    # Views one element into a larger buffer: 4-byte aligned, not 16.
    T = 301
    d = inputs("td_lambda", N, T, seed=3500)
    s = f32_scalars("td_lambda", synthetic.SCALARS["td_lambda"])
    dt = transpose(d)

    def shifted(a):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
        if a.ndim == 1:
            return t
        big = torch.zeros(a.size + 1, dtype=t.dtype, device="cuda")
        big[1:] = t.reshape(-1)
        return big[1:].view(a.shape)

    t = {k: shifted(v) for k, v in dt.items()}
    out = slr.rlscan_td_lambda_tm(t["rewards"], t["values"], t["bootstrap"], t["terminated"], t["truncated"],
                                  t["trunc_value"], **s)
    ref = oracle_run("td_lambda", d, **s)
    assert_parity("td_lambda", (np.ascontiguousarray(out.cpu().numpy().T),), ref, what="unaligned views")


def test_time_major_graph_replay():
    # Tickets wrap and the epoch advances on the device: a captured call can
    # be replayed any number of times.
    N, T = 96, 3000
    d = inputs("gae", N, T, seed=3600)
    s = f32_scalars("gae", synthetic.SCALARS["gae"])
    dt = transpose(d)
    t = {k: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in dt.items()}
    adv = torch.empty((T, N), dtype=torch.float32, device="cuda")
    ret = torch.empty_like(adv)
    info = slr.rlscan_query_plan_tm("gae", N, T)
    assert info["lookback"] == 1
    st = torch.cuda.Stream()
    slr.rlscan_reserve_workspace(info["workspace_bytes"], stream=st)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        slr.rlscan_gae_tm(t["rewards"], t["values"], t["bootstrap"], t["terminated"], t["truncated"],
                          t["trunc_value"], advantages=adv, returns=ret, stream=st, **s)
    ref = oracle_run("gae", d, **s)
    for _ in range(5):
        adv.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert_parity("gae", (np.ascontiguousarray(adv.cpu().numpy().T), np.ascontiguousarray(ret.cpu().numpy().T)),
                      ref, what="graph replay")
    assert slr.rlscan_sync_status() == 0


def test_time_major_withheld_carry_times_out_and_reports(options):
    # 32 environments of 4000 steps: 63 chunks along T.  The block holding
    # the first ticket (the last chunk in time) never publishes; the chunk
    # before it waits 20 ms per environment, gives up and reports.
    options("lookback_timeout_ns", 20_000_000)
    options("test_starve_lookback", 1)
    N, T = 32, 4000
    d = synthetic.make_inputs("discounted_return", N, T, seed=3700, p_term=0.0)
    s = f32_scalars("discounted_return", synthetic.SCALARS["discounted_return"])
    assert slr.rlscan_sync_status() == 0
    tm_run("discounted_return", transpose(d), **s)
    assert slr.rlscan_sync_status() == 4  # RLSCAN_ERR_TIMEOUT
    options("test_starve_lookback", 0)
    check_tm("discounted_return", N, T, seed=3700, what="after timeout")
    assert slr.rlscan_sync_status() == 0


def test_time_major_plan_shapes():
    # One block covers T <= 64 with 1..8 time slices; longer windows chain.
    assert slr.rlscan_query_plan_tm("gae", 4096, 512)["lookback"] == 1
    for T, slices in [(1, 1), (8, 1), (9, 2), (16, 2), (32, 4), (64, 8)]:
        info = slr.rlscan_query_plan_tm("gae", 1000, T)
        assert info["lookback"] == 0
        assert info["chunks"] == -(-1000 // (256 // slices))


@pytest.mark.parametrize("est", TM_ESTIMATORS + ("affine_scan",))
def test_transposed_views_take_the_time_major_kernel(est):
    # [N, T] views of time-major [T, N] storage (buf.T) go to the time-major
    # kernel without a copy; results come back as [N, T] views.
    N, T = 96, 700
    d = inputs(est, N, T, seed=3800)
    s = f32_scalars(est, dict(synthetic.SCALARS.get(est, {})))
    views = {k: None if v is None else (torch.from_numpy(np.ascontiguousarray(v)).cuda() if k in PER_ENV
                                        else torch.from_numpy(np.ascontiguousarray(v)).cuda().T)
             for k, v in transpose(d).items()}
    args = {"gae": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
            "vtrace": ("log_rhos", "rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
            "td_lambda": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
            "discounted_return": ("rewards", "bootstrap", "terminated", "truncated", "trunc_value"),
            "elig_trace": ("inputs", "init_trace", "terminated", "truncated"),
            "episodic_prefix_sum": ("x", "terminated", "truncated"),
            "affine_scan": ("a", "b", "reset", "init")}[est]
    kw = {} if est == "episodic_prefix_sum" else dict(s)
    if est == "affine_scan":
        kw = {"reverse": bool(s.get("reverse", False))}
    for k, v in views.items():
        if k not in PER_ENV and v is not None:
            assert not v.is_contiguous() and v.shape == (N, T)
    res = getattr(slr, f"rlscan_{est}")(*[views.get(k) for k in args], **kw)
    res = res if isinstance(res, tuple) else (res,)
    for r in res:
        assert r is None or (r.shape == (N, T) and r.t().is_contiguous())
    got = tuple(None if r is None else r.cpu().numpy() for r in res)
    assert_parity(est, got, oracle_run(est, d, **s), what="transposed views")
