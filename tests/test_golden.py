"""Hand-worked examples (tests/golden/worked_examples.json): every
intermediate step is written out in the fixture, from the estimators'
definitions and the pages' boundary rules.  The oracle must reproduce them
(CPU); the kernels must too (GPU, fp32 tolerance)."""
import json
import os

import numpy as np
import pytest

import oracle

from .util import OUTPUT_NAMES, TOL

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_examples.json")
EXAMPLES = json.load(open(GOLDEN))["examples"]
INT_KEYS = {"actions": np.int32, "x": np.int32}
FLAG_KEYS = ("terminated", "truncated", "reset")
OPTIONAL = {"gae": ("truncated", "trunc_value"), "vtrace": ("truncated", "trunc_value"),
            "td_lambda": ("truncated", "trunc_value"), "discounted_return": ("truncated", "trunc_value"),
            "retrace": ("truncated", "trunc_value"), "elig_trace": ("truncated", "init_trace"),
            "episodic_prefix_sum": ("truncated",), "affine_scan": ("reset", "init")}


def arrays(ex):
    d = {}
    for k, v in ex["inputs"].items():
        dt = np.uint8 if k in FLAG_KEYS else INT_KEYS.get(k, np.float32)
        d[k] = np.ascontiguousarray(np.array(v, dtype=np.float64).astype(dt))
    for k in OPTIONAL[ex["estimator"]]:
        d.setdefault(k, None)
    return d


def compare(ex, got, tol):
    for name, g in zip(OUTPUT_NAMES[ex["estimator"]], got):
        want = np.array(ex["expected"][name], dtype=np.float64)
        g = np.asarray(g, dtype=np.float64)
        assert g.shape == want.shape, (ex["name"], name, g.shape)
        err = np.abs(g - want)
        assert (err <= tol * (1.0 + np.abs(want))).all(), (ex["name"], name, g.tolist(), want.tolist())


@pytest.mark.parametrize("ex", EXAMPLES, ids=[e["name"] for e in EXAMPLES])
def test_oracle_reproduces_worked_example(ex):
    got = oracle.run(ex["estimator"], arrays(ex), **ex["scalars"])
    got = got if isinstance(got, tuple) else (got,)
    compare(ex, got, ex.get("tolerance", 1e-12))


@pytest.mark.gpu
@pytest.mark.parametrize("ex", EXAMPLES, ids=[e["name"] for e in EXAMPLES])
def test_kernels_reproduce_worked_example(ex):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from .util import gpu_run
    scal = dict(ex["scalars"])
    if ex["estimator"] == "affine_scan":
        scal["reverse"] = bool(scal.get("reverse", False))
    got = gpu_run(ex["estimator"], arrays(ex), **scal)
    compare(ex, got, max(TOL, ex.get("tolerance", 0.0)))
