"""Shared helpers for the GPU parity tests: run an estimator through the C ABI
(via the Python binding) and through the CPU oracle on the same host arrays,
and compare them."""
import numpy as np

import oracle

TOL = 1e-4  # |gpu - ref| <= TOL * (1 + |ref|) for fp32 outputs; int32 outputs bit-exact

OUTPUT_NAMES = {
    "gae": ("advantages", "returns"),
    "vtrace": ("vs", "pg_advantages"),
    "retrace": ("q_ret",),
    "td_lambda": ("returns",),
    "discounted_return": ("returns",),
    "elig_trace": ("traces",),
    "episodic_prefix_sum": ("out",),
    "affine_scan": ("x",),
}


def f32(x):
    """The fp32-rounded value of a scalar, as the GPU sees it."""
    return float(np.float32(x))


def to_dev(d, device="cuda"):
    import torch
    out = {}
    for k, v in d.items():
        out[k] = None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device)
    return out


def gpu_run(est, d, stream=None, **scal):
    """Run one estimator on the GPU; returns a tuple of numpy outputs."""
    import segmented_linear_recurrence_b200 as slr
    t = to_dev(d)
    if est == "gae":
        res = slr.rlscan_gae(t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                             t.get("truncated"), t.get("trunc_value"), stream=stream, **scal)
    elif est == "vtrace":
        res = slr.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["bootstrap"],
                                t["terminated"], t.get("truncated"), t.get("trunc_value"),
                                stream=stream, **scal)
    elif est == "retrace":
        res = slr.rlscan_retrace(t["q"], t["pi"], t["mu_a"], t["actions"], t["rewards"],
                                 t["bootstrap"], t["terminated"], t.get("truncated"),
                                 t.get("trunc_value"), stream=stream, **scal)
    elif est == "td_lambda":
        res = slr.rlscan_td_lambda(t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                                   t.get("truncated"), t.get("trunc_value"), stream=stream, **scal)
    elif est == "discounted_return":
        res = slr.rlscan_discounted_return(t["rewards"], t.get("bootstrap"), t["terminated"],
                                           t.get("truncated"), t.get("trunc_value"), stream=stream,
                                           **scal)
    elif est == "elig_trace":
        res = slr.rlscan_elig_trace(t["inputs"], t.get("init_trace"), t["terminated"],
                                    t.get("truncated"), stream=stream, **scal)
    elif est == "episodic_prefix_sum":
        res = slr.rlscan_episodic_prefix_sum(t["x"], t["terminated"], t.get("truncated"),
                                             stream=stream)
    elif est == "affine_scan":
        res = slr.rlscan_affine_scan(t["a"], t["b"], t.get("reset"), t.get("init"),
                                     reverse=bool(scal.get("reverse", False)), stream=stream)
    else:
        raise ValueError(est)
    res = res if isinstance(res, tuple) else (res,)
    return tuple(None if r is None else r.cpu().numpy() for r in res)


def oracle_run(est, d, **scal):
    kw = dict(scal)
    res = oracle.run(est, d, **kw)
    if est == "episodic_prefix_sum":
        return (res[0],)
    return res if isinstance(res, tuple) else (res,)


def f32_scalars(est, scal):
    """The fp32-rounded scalars, so both sides see the same gamma / lambda / clips."""
    return {k: f32(v) for k, v in scal.items()}


def assert_parity(est, gpu, ref, tol=TOL, what=""):
    for name, g, r in zip(OUTPUT_NAMES[est], gpu, ref):
        if g is None:
            continue
        assert g.shape == r.shape, (name, g.shape, r.shape)
        if est == "episodic_prefix_sum":
            np.testing.assert_array_equal(g, r, err_msg=f"{est}.{name} {what}")
            continue
        r64 = r.astype(np.float64)
        err = np.abs(g.astype(np.float64) - r64)
        bound = tol * (1.0 + np.abs(r64))
        bad = ~(err <= bound)
        if bad.any():
            idx = np.argwhere(bad)[:5]
            worst = float((err / bound).max())
            raise AssertionError(
                f"{est}.{name} {what}: {int(bad.sum())} of {bad.size} outside "
                f"{tol}*(1+|ref|); worst ratio {worst:.3g}; first bad {idx.tolist()} "
                f"gpu={g[tuple(idx[0])]} ref={r[tuple(idx[0])]}")


def check(est, d, scal=None, tol=TOL, what=""):
    scal = dict(scal if scal is not None else {})
    s32 = f32_scalars(est, scal)
    gpu = gpu_run(est, d, **s32)
    ref = oracle_run(est, d, **s32)
    assert_parity(est, gpu, ref, tol=tol, what=what)
    return gpu, ref
