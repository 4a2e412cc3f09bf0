"""GPU parity: librlscan (through its C ABI) against the fp64 CPU oracle.

Every named workload runs at full size in the same launch configuration the
benchmark times (the library's default plan), and the whole output is
compared element by element: fp32 outputs within 1e-4 * (1 + |ref|), the
int32 episodic prefix sum bit-exact.  Edge cases cover ragged and tiny rows,
rows longer than one block (decoupled look-back), flag patterns at the row
edges, degenerate scalars and unaligned buffers.
"""
import numpy as np
import pytest
import torch

from segmented_linear_recurrence_b200 import synthetic
from segmented_linear_recurrence_b200 import build as slr_build

from .util import assert_parity, check, f32_scalars, gpu_run, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()


def _cases():
    out = []
    for wl, w in synthetic.WORKLOADS.items():
        for est in w["estimators"]:
            for T in w["Ts"]:
                out.append(pytest.param(wl, est, T, id=f"{wl}-{est}-T{T}"))
    return out


@pytest.mark.parametrize("workload,est,T", _cases())
def test_workload_parity(workload, est, T):
    d = synthetic.workload_inputs(workload, est, T)
    check(est, d, synthetic.SCALARS[est], what=f"{workload} T={T}")


EDGE_T = [1, 2, 3, 4, 5, 31, 33, 127, 129, 1000, 4097]


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
@pytest.mark.parametrize("T", EDGE_T)
def test_ragged_rows(est, T):
    N = 7 if T < 1000 else 3
    d = synthetic.make_inputs(est, N, T, seed=500 + T, p_term=0.05, p_trunc=0.05, A=5,
                              with_init=True)
    check(est, d, synthetic.SCALARS[est], what=f"N={N} T={T}")


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_single_long_row(est):
    # one row much longer than a block's chunk: many chunks chained by look-back
    T = 100_003 if est != "retrace" else 20_011
    d = synthetic.make_inputs(est, 1, T, seed=77, p_term=0.0005, p_trunc=0.0005, A=6,
                              with_init=True)
    check(est, d, synthetic.SCALARS[est], what=f"N=1 T={T}")


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
@pytest.mark.parametrize("pattern", ["no_done", "all_done", "done_at_edges", "term_and_trunc"])
def test_flag_patterns(est, pattern):
    N, T = 9, 64
    d = synthetic.make_inputs(est, N, T, seed=61, p_term=0.0, p_trunc=0.1, A=4, with_init=True)
    term = np.zeros((N, T), np.uint8)
    trunc = d["truncated"]
    if pattern == "all_done":
        term[:] = 1
    elif pattern == "done_at_edges":
        term[:, 0] = 1
        term[:, T - 1] = 1
        trunc[:] = 0
        trunc[:, 1] = 1
        trunc[:, T - 2] = 1
    elif pattern == "term_and_trunc":
        term[:, ::3] = 1
        trunc[:, ::2] = 1
    d["terminated"] = term
    check(est, d, synthetic.SCALARS[est], what=pattern)


@pytest.mark.parametrize("est", ["gae", "vtrace", "retrace", "td_lambda", "discounted_return",
                                 "elig_trace"])
@pytest.mark.parametrize("gamma,lam", [(0.0, 0.95), (0.99, 0.0), (0.99, 1.0), (1.0, 1.0)])
def test_degenerate_scalars(est, gamma, lam):
    d = synthetic.make_inputs(est, 33, 257, seed=62, p_term=0.02, p_trunc=0.01, A=3)
    scal = dict(synthetic.SCALARS[est])
    scal["gamma"] = gamma
    if "lam" in scal:
        scal["lam"] = lam
    check(est, d, scal, what=f"gamma={gamma} lam={lam}")


def test_vtrace_clipping_thresholds():
    d = synthetic.make_inputs("vtrace", 64, 300, seed=63, p_term=0.01, p_trunc=0.01)
    d["log_rhos"] = (d["log_rhos"] * 5).astype(np.float32)
    check("vtrace", d, dict(gamma=0.97, lam=0.9, rho_bar=1.5, c_bar=0.8), what="clips")


def test_optional_outputs_and_inputs():
    import segmented_linear_recurrence_b200 as slr
    d = synthetic.make_inputs("gae", 16, 96, seed=64, p_term=0.05)
    t = {k: (None if v is None else torch.from_numpy(v).cuda()) for k, v in d.items()}
    adv, ret = slr.rlscan_gae(t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                              want_returns=False)
    assert ret is None
    ref, _ = oracle_run("gae", d, **f32_scalars("gae", synthetic.SCALARS["gae"]))
    assert_parity("gae", (adv.cpu().numpy(), None), (ref, None))
    # no termination array at all
    d2 = dict(d, terminated=np.zeros_like(d["terminated"]))
    g = slr.rlscan_gae(t["rewards"], t["values"], t["bootstrap"], None)
    r2 = oracle_run("gae", d2, **f32_scalars("gae", synthetic.SCALARS["gae"]))
    assert_parity("gae", tuple(x.cpu().numpy() for x in g), r2)
    # discounted return without bootstrap
    d3 = synthetic.make_inputs("discounted_return", 16, 96, seed=65, p_term=0.05, with_bootstrap=False)
    check("discounted_return", d3, {"gamma": 0.9})


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_unaligned_buffers_take_the_scalar_path(est):
    # views that start one element into a larger buffer: 4-byte aligned only
    N, T = 11, 203
    d = synthetic.make_inputs(est, N, T, seed=66, p_term=0.03, p_trunc=0.03, A=5, with_init=True)
    import segmented_linear_recurrence_b200 as slr
    dev = {}
    for k, v in d.items():
        if v is None:
            continue
        flat = torch.from_numpy(np.ascontiguousarray(v).reshape(-1))
        big = torch.zeros(flat.numel() + 1, dtype=flat.dtype, device="cuda")
        big[1:] = flat.cuda()
        dev[k] = big[1:].view(v.shape)
    scal = f32_scalars(est, synthetic.SCALARS[est])
    fn = getattr(slr, f"rlscan_{est}")
    if est == "gae":
        res = fn(dev["rewards"], dev["values"], dev["bootstrap"], dev["terminated"],
                 dev.get("truncated"), dev.get("trunc_value"), **scal)
    elif est == "vtrace":
        res = fn(dev["log_rhos"], dev["rewards"], dev["values"], dev["bootstrap"], dev["terminated"],
                 dev.get("truncated"), dev.get("trunc_value"), **scal)
    elif est == "retrace":
        res = fn(dev["q"], dev["pi"], dev["mu_a"], dev["actions"], dev["rewards"], dev["bootstrap"],
                 dev["terminated"], dev.get("truncated"), dev.get("trunc_value"), **scal)
    elif est == "td_lambda":
        res = fn(dev["rewards"], dev["values"], dev["bootstrap"], dev["terminated"],
                 dev.get("truncated"), dev.get("trunc_value"), **scal)
    elif est == "discounted_return":
        res = fn(dev["rewards"], dev.get("bootstrap"), dev["terminated"], dev.get("truncated"),
                 dev.get("trunc_value"), **scal)
    elif est == "elig_trace":
        res = fn(dev["inputs"], dev.get("init_trace"), dev["terminated"], dev.get("truncated"), **scal)
    else:
        res = fn(dev["x"], dev["terminated"], dev.get("truncated"))
    res = res if isinstance(res, tuple) else (res,)
    gpu = tuple(None if r is None else r.cpu().numpy() for r in res)
    assert_parity(est, gpu, oracle_run(est, d, **scal), what="unaligned")


def test_invalid_action_is_reported_not_read():
    import segmented_linear_recurrence_b200 as slr
    d = synthetic.make_inputs("retrace", 4, 40, seed=67, A=5)
    d["actions"][2, 7] = 5  # out of [0, A)
    d["actions"][3, 39] = -1
    t = {k: (None if v is None else torch.from_numpy(v).cuda()) for k, v in d.items()}
    assert slr.rlscan_sync_status() == 0
    slr.rlscan_retrace(t["q"], t["pi"], t["mu_a"], t["actions"], t["rewards"], t["bootstrap"],
                       t["terminated"])
    assert slr.rlscan_sync_status() == 1  # RLSCAN_ERR_INVALID_ARG
    assert slr.rlscan_sync_status() == 0  # cleared


@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_host_tensors_round_trip(est):
    # the public API also takes (pinned) host tensors: copies in, kernel, copies out
    d = synthetic.make_inputs(est, 32, 130, seed=68, p_term=0.02, p_trunc=0.02, A=4)
    import segmented_linear_recurrence_b200 as slr
    h = {k: (None if v is None else torch.from_numpy(v).pin_memory()) for k, v in d.items()}
    scal = f32_scalars(est, synthetic.SCALARS[est])
    fn = getattr(slr, f"rlscan_{est}")
    args = {
        "gae": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
        "vtrace": ("log_rhos", "rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
        "retrace": ("q", "pi", "mu_a", "actions", "rewards", "bootstrap", "terminated", "truncated",
                    "trunc_value"),
        "td_lambda": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
        "discounted_return": ("rewards", "bootstrap", "terminated", "truncated", "trunc_value"),
        "elig_trace": ("inputs", "init_trace", "terminated", "truncated"),
        "episodic_prefix_sum": ("x", "terminated", "truncated"),
    }[est]
    res = fn(*[h.get(a) for a in args], **({} if est == "episodic_prefix_sum" else scal))
    res = res if isinstance(res, tuple) else (res,)
    for r in res:
        assert r is None or not r.is_cuda
    gpu = tuple(None if r is None else r.numpy() for r in res)
    assert_parity(est, gpu, oracle_run(est, d, **scal), what="host tensors")


def test_repeated_calls_are_bit_identical():
    # the combine order is fixed by the launch shape, never by timing
    d = synthetic.make_inputs("vtrace", 64, 16384, seed=69, p_term=0.001, p_trunc=0.001)
    s = f32_scalars("vtrace", synthetic.SCALARS["vtrace"])
    first = gpu_run("vtrace", d, **s)
    for _ in range(5):
        again = gpu_run("vtrace", d, **s)
        for a, b in zip(first, again):
            np.testing.assert_array_equal(a, b)
