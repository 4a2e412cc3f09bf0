"""Seeded synthetic rollout generators shared by the tests, the smoke check and
the benchmark.

This module draws random inputs only: it holds none of the estimators'
arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any computation.  Every array is numpy on the host, row-major
``[N, T]`` (Retrace's ``q`` / ``pi``: ``[N, T, A]``), with the dtypes the
C ABI takes: float32 values, uint8 flags (0/1), int32 actions / integers.

The distributions follow the workloads the rl-triton pages benchmark
("thousands of environments, short rollouts"; per-step termination and
optional truncation with an appended bootstrap value): rewards, values and
bootstrap values ~ N(0, 1); terminated ~ Bernoulli(p_term); truncated ~
Bernoulli(p_trunc) with a dense trunc_value ~ N(0, 1) (read only where
truncated); V-trace log-ratios ~ N(0, 0.3^2); eligibility inputs ~ N(0, 1);
prefix-sum integers uniform in [-100, 100]; Retrace Q ~ N(0, 1), pi =
softmax of N(0, 1) logits over A actions, behaviour probability of the taken
action mu(a_t) ~ U(0.05, 1], actions uniform in [0, A).
"""
from __future__ import annotations

import numpy as np

ESTIMATORS = ("gae", "vtrace", "retrace", "td_lambda", "discounted_return", "elig_trace",
              "episodic_prefix_sum")

# Scalars each estimator is run with in the named workloads.
SCALARS = {
    "gae": dict(gamma=0.99, lam=0.95),
    "td_lambda": dict(gamma=0.99, lam=0.95),
    "discounted_return": dict(gamma=0.99),
    "vtrace": dict(gamma=0.99, lam=1.0, rho_bar=1.0, c_bar=1.0),
    "retrace": dict(gamma=0.99, lam=0.95),
    "elig_trace": dict(gamma=0.99, lam=0.95),
    "episodic_prefix_sum": dict(),
    "affine_scan": dict(reverse=True),
}

SWEEP_T = (32, 64, 128, 256, 512, 1024, 2048)

# The named workloads.  index -> seed base.
WORKLOADS = {
    "gae_64x32": dict(index=0, N=64, Ts=(32,), estimators=("gae",), p_term=0.02, p_trunc=0.0),
    "all7_4096x128": dict(index=1, N=4096, Ts=(128,), estimators=ESTIMATORS, p_term=0.01,
                          p_trunc=0.0, A=18),
    "sweep_4096xT": dict(index=2, N=4096, Ts=SWEEP_T,
                         estimators=("gae", "vtrace", "td_lambda", "discounted_return"),
                         p_term=0.02, p_trunc=0.005),
    "retrace_2048x512x18": dict(index=3, N=2048, Ts=(512,), estimators=("retrace",), p_term=0.01,
                                p_trunc=0.0, A=18),
    "long_256x16384": dict(index=4, N=256, Ts=(16384,), estimators=ESTIMATORS, p_term=0.01,
                           p_trunc=0.0, A=6),
    # the generic affine scan (backward), resets at p_term
    "affine_4096xT": dict(index=5, N=4096, Ts=(512, 2048), estimators=("affine_scan",), p_term=0.01,
                          p_trunc=0.0),
    # GAE with bfloat16 I/O (inputs rounded to bf16 on the device side)
    "gae_bf16_4096xT": dict(index=7, N=4096, Ts=(512, 2048), estimators=("gae",), p_term=0.02, p_trunc=0.005,
                            io="bf16"),
    # the sweep's estimators and the affine scan on time-major [T, N] buffers
    "tm_4096xT": dict(index=6, N=4096, Ts=(512, 2048),
                      estimators=("gae", "vtrace", "td_lambda", "discounted_return", "affine_scan"),
                      p_term=0.02, p_trunc=0.005, layout="time_major"),
}

# Per-environment arrays ([N]) keep their shape in the time-major layout.
PER_ENV_KEYS = ("bootstrap", "init_trace", "init")


def to_time_major(d: dict) -> dict:
    """The same inputs with every [N, T] array stored time-major [T, N]."""
    return {k: (None if v is None else (v if k in PER_ENV_KEYS else np.ascontiguousarray(v.T)))
            for k, v in d.items()}


def seed_for(workload: str, estimator: str, T: int) -> int:
    w = WORKLOADS[workload]
    k = ESTIMATORS.index(estimator) if estimator in ESTIMATORS else len(ESTIMATORS)
    return 1000 + 100 * w["index"] + 10 * list(w["Ts"]).index(T) + k


def _normal(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32)


def _bern(rng, shape, p):
    return (rng.random(shape, dtype=np.float32) < np.float32(p)).astype(np.uint8)


def make_inputs(estimator: str, N: int, T: int, *, seed: int, p_term: float = 0.01,
                p_trunc: float = 0.0, A: int = 18, with_init: bool = False,
                with_bootstrap: bool = True) -> dict:
    """Draw one estimator's inputs.  Keys match the API's parameter names."""
    if estimator not in ESTIMATORS:
        raise ValueError(f"unknown estimator {estimator!r}")
    rng = np.random.Generator(np.random.PCG64(seed))
    shp = (N, T)
    d: dict = {}
    if estimator in ("gae", "td_lambda", "vtrace"):
        d["rewards"] = _normal(rng, shp)
        d["values"] = _normal(rng, shp)
        d["bootstrap"] = _normal(rng, (N,))
        if estimator == "vtrace":
            d["log_rhos"] = (np.float32(0.3) * _normal(rng, shp)).astype(np.float32)
    elif estimator == "discounted_return":
        d["rewards"] = _normal(rng, shp)
        d["bootstrap"] = _normal(rng, (N,)) if with_bootstrap else None
    elif estimator == "retrace":
        d["q"] = _normal(rng, (N, T, A))
        logits = _normal(rng, (N, T, A)).astype(np.float64)
        logits -= logits.max(axis=-1, keepdims=True)
        e = np.exp(logits)
        d["pi"] = (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)
        d["actions"] = rng.integers(0, A, size=shp, dtype=np.int32)
        # U(0.05, 1]: 1 - U[0, 0.95)
        d["mu_a"] = (np.float32(1.0) - np.float32(0.95) * rng.random(shp, dtype=np.float32))
        d["rewards"] = _normal(rng, shp)
        d["bootstrap"] = _normal(rng, (N,))
    elif estimator == "elig_trace":
        d["inputs"] = _normal(rng, shp)
        d["init_trace"] = _normal(rng, (N,)) if with_init else None
    elif estimator == "episodic_prefix_sum":
        d["x"] = rng.integers(-100, 101, size=shp, dtype=np.int32)
    d["terminated"] = _bern(rng, shp, p_term)
    if p_trunc > 0.0:
        d["truncated"] = _bern(rng, shp, p_trunc)
        if estimator not in ("elig_trace", "episodic_prefix_sum"):
            d["trunc_value"] = _normal(rng, shp)
    else:
        d["truncated"] = None
        if estimator not in ("elig_trace", "episodic_prefix_sum"):
            d["trunc_value"] = None
    return d


def workload_inputs(workload: str, estimator: str, T: int | None = None) -> dict:
    """Inputs of one estimator in a named workload (first T if not given)."""
    w = WORKLOADS[workload]
    T = w["Ts"][0] if T is None else T
    if estimator == "affine_scan":
        return make_affine_inputs(w["N"], T, seed=seed_for(workload, estimator, T), p_reset=w["p_term"])
    return make_inputs(estimator, w["N"], T, seed=seed_for(workload, estimator, T),
                       p_term=w["p_term"], p_trunc=w["p_trunc"], A=w.get("A", 18))


def input_bytes(d: dict) -> int:
    return int(sum(v.nbytes for v in d.values() if isinstance(v, np.ndarray)))


def make_affine_inputs(N: int, T: int, *, seed: int, p_reset: float = 0.01, with_init: bool = True,
                       a_low: float = 0.8, a_high: float = 1.0) -> dict:
    """Seeded inputs of the generic affine scan: a ~ U(a_low, a_high) (decay
    factors such as gamma * lambda), b ~ N(0, 1), reset ~ Bernoulli(p_reset)
    (uint8, None when p_reset is 0), init ~ N(0, 1) per row (or None)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    a = rng.uniform(a_low, a_high, size=(N, T)).astype(np.float32)
    b = _normal(rng, (N, T))
    reset = (rng.random((N, T)) < p_reset).astype(np.uint8) if p_reset > 0 else None
    init = _normal(rng, (N,)) if with_init else None
    return {"a": a, "b": b, "reset": reset, "init": init}
