"""ctypes front end of the fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference leg may import this module.  The product library
(librlscan) never loads it, and it loads nothing from the product.

Each function takes numpy host arrays (fp32 / uint8 / int32, row-major
``[N, T]``; Retrace's ``q`` and ``pi`` are ``[N, T, A]``) and returns fp64
numpy arrays computed by the sequential loops in ``rlscan_oracle.c``.
Scalars (gamma, lambda, rho_bar, c_bar) are passed as doubles; callers that
compare against the fp32 GPU path pass the fp32-rounded value.
"""
from __future__ import annotations

import ctypes
import inspect

import numpy as np

from . import build as _build

_lib = None


def bind(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    sig = {
        "rlo_gae": [i64, i64, vp, vp, vp, vp, vp, vp, dbl, dbl, vp, vp],
        "rlo_td_lambda": [i64, i64, vp, vp, vp, vp, vp, vp, dbl, dbl, vp],
        "rlo_discounted_return": [i64, i64, vp, vp, vp, vp, vp, dbl, vp],
        "rlo_vtrace": [i64, i64, vp, vp, vp, vp, vp, vp, vp, dbl, dbl, dbl, dbl, vp, vp],
        "rlo_retrace": [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, dbl, dbl, vp],
        "rlo_elig_trace": [i64, i64, vp, vp, vp, vp, dbl, dbl, vp],
        "rlo_episodic_prefix_sum": [i64, i64, vp, vp, vp, vp, vp],
        "rlo_affine_scan": [i64, i64, vp, vp, vp, vp, ctypes.c_int, vp],
        "rlo_affine_scan_grad": [i64, i64, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp],
        "rlo_affine_scan_tm": [i64, i64, vp, vp, vp, vp, ctypes.c_int, vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(_build.build()))
    return _lib


def _p(a, dtype):
    """Pointer to a C-contiguous array of the given dtype (None -> NULL)."""
    if a is None:
        return None, None
    arr = np.ascontiguousarray(a, dtype=dtype)
    return arr, arr.ctypes.data_as(ctypes.c_void_p)


def _dims(x):
    x = np.asarray(x)
    if x.ndim != 2:
        raise ValueError("per-step arrays must be 2-D [N, T]")
    return int(x.shape[0]), int(x.shape[1])


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments (rc={rc})")


def gae(rewards, values, bootstrap, terminated, truncated=None, trunc_value=None,
        gamma=0.99, lam=0.95):
    N, T = _dims(rewards)
    keep = [_p(rewards, np.float32), _p(values, np.float32), _p(bootstrap, np.float32),
            _p(terminated, np.uint8), _p(truncated, np.uint8), _p(trunc_value, np.float32)]
    adv = np.empty((N, T), np.float64)
    ret = np.empty((N, T), np.float64)
    rc = _load().rlo_gae(N, T, *[k[1] for k in keep], float(gamma), float(lam),
                         adv.ctypes.data_as(ctypes.c_void_p), ret.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "gae")
    return adv, ret


def td_lambda(rewards, values, bootstrap, terminated, truncated=None, trunc_value=None,
              gamma=0.99, lam=0.95):
    N, T = _dims(rewards)
    keep = [_p(rewards, np.float32), _p(values, np.float32), _p(bootstrap, np.float32),
            _p(terminated, np.uint8), _p(truncated, np.uint8), _p(trunc_value, np.float32)]
    out = np.empty((N, T), np.float64)
    rc = _load().rlo_td_lambda(N, T, *[k[1] for k in keep], float(gamma), float(lam),
                               out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "td_lambda")
    return out


def discounted_return(rewards, bootstrap, terminated, truncated=None, trunc_value=None,
                      gamma=0.99):
    N, T = _dims(rewards)
    keep = [_p(rewards, np.float32), _p(bootstrap, np.float32), _p(terminated, np.uint8),
            _p(truncated, np.uint8), _p(trunc_value, np.float32)]
    out = np.empty((N, T), np.float64)
    rc = _load().rlo_discounted_return(N, T, *[k[1] for k in keep], float(gamma),
                                       out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "discounted_return")
    return out


def vtrace(log_rhos, rewards, values, bootstrap, terminated, truncated=None, trunc_value=None,
           gamma=0.99, lam=1.0, rho_bar=1.0, c_bar=1.0):
    N, T = _dims(rewards)
    keep = [_p(log_rhos, np.float32), _p(rewards, np.float32), _p(values, np.float32),
            _p(bootstrap, np.float32), _p(terminated, np.uint8), _p(truncated, np.uint8),
            _p(trunc_value, np.float32)]
    vs = np.empty((N, T), np.float64)
    pg = np.empty((N, T), np.float64)
    rc = _load().rlo_vtrace(N, T, *[k[1] for k in keep], float(gamma), float(lam),
                            float(rho_bar), float(c_bar), vs.ctypes.data_as(ctypes.c_void_p),
                            pg.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "vtrace")
    return vs, pg


def retrace(q, pi, mu_a, actions, rewards, bootstrap, terminated, truncated=None,
            trunc_value=None, gamma=0.99, lam=0.95):
    q = np.asarray(q)
    if q.ndim != 3:
        raise ValueError("q must be [N, T, A]")
    N, T, A = (int(s) for s in q.shape)
    keep = [_p(q, np.float32), _p(pi, np.float32), _p(mu_a, np.float32), _p(actions, np.int32),
            _p(rewards, np.float32), _p(bootstrap, np.float32), _p(terminated, np.uint8),
            _p(truncated, np.uint8), _p(trunc_value, np.float32)]
    out = np.empty((N, T), np.float64)
    rc = _load().rlo_retrace(N, T, A, *[k[1] for k in keep], float(gamma), float(lam),
                             out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "retrace")
    return out


def elig_trace(inputs, init_trace, terminated, truncated=None, gamma=0.99, lam=0.95):
    N, T = _dims(inputs)
    keep = [_p(inputs, np.float32), _p(init_trace, np.float32), _p(terminated, np.uint8),
            _p(truncated, np.uint8)]
    out = np.empty((N, T), np.float64)
    rc = _load().rlo_elig_trace(N, T, *[k[1] for k in keep], float(gamma), float(lam),
                                out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "elig_trace")
    return out


def episodic_prefix_sum(x, terminated, truncated=None):
    """Returns (int32 sums, max |S| over all steps computed in int64)."""
    N, T = _dims(x)
    keep = [_p(x, np.int32), _p(terminated, np.uint8), _p(truncated, np.uint8)]
    out = np.empty((N, T), np.int32)
    mx = ctypes.c_int64(0)
    rc = _load().rlo_episodic_prefix_sum(N, T, *[k[1] for k in keep],
                                         out.ctypes.data_as(ctypes.c_void_p),
                                         ctypes.cast(ctypes.pointer(mx), ctypes.c_void_p))
    _check(rc, "episodic_prefix_sum")
    return out, int(mx.value)


def affine_scan(a, b, reset=None, init=None, reverse=False):
    """x_t = b_t + a_t x_prev in scan order (backward when `reverse`), x_prev
    = init[n] (None: 0) at the row's first step, x_t = b_t where reset."""
    N, T = _dims(a)
    keep = [_p(a, np.float32), _p(b, np.float32), _p(reset, np.uint8), _p(init, np.float32)]
    out = np.empty((N, T), np.float64)
    rc = _load().rlo_affine_scan(N, T, *[k[1] for k in keep], 1 if reverse else 0,
                                 out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "affine_scan")
    return out


def affine_scan_tm(a, b, reset=None, init=None, reverse=False):
    """affine_scan on time-major [T, N] arrays (init [N]); returns [T, N]."""
    a = np.asarray(a)
    if a.ndim != 2:
        raise ValueError("time-major arrays must be 2-D [T, N]")
    T, N = int(a.shape[0]), int(a.shape[1])
    keep = [_p(a, np.float32), _p(b, np.float32), _p(reset, np.uint8), _p(init, np.float32)]
    out = np.empty((T, N), np.float64)
    rc = _load().rlo_affine_scan_tm(N, T, *[k[1] for k in keep], 1 if reverse else 0,
                                    out.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "affine_scan_tm")
    return out


def affine_scan_grad(a, x, dy, reset=None, init=None, reverse=False):
    """Adjoint of affine_scan: returns (da, db, dinit) for upstream dy, given
    the forward output x (all fp64)."""
    N, T = _dims(a)
    keep = [_p(a, np.float32), _p(x, np.float32), _p(dy, np.float32), _p(reset, np.uint8),
            _p(init, np.float32)]
    da = np.empty((N, T), np.float64)
    db = np.empty((N, T), np.float64)
    dinit = np.empty((N,), np.float64)
    rc = _load().rlo_affine_scan_grad(N, T, *[k[1] for k in keep], 1 if reverse else 0,
                                      da.ctypes.data_as(ctypes.c_void_p), db.ctypes.data_as(ctypes.c_void_p),
                                      dinit.ctypes.data_as(ctypes.c_void_p))
    _check(rc, "affine_scan_grad")
    return da, db, dinit


# Convenience: dispatch by estimator name on a dict of inputs as produced by
# segmented_linear_recurrence_b200.synthetic (keys match parameter names).
def run(name, inp, **scal):
    fn = {"gae": gae, "td_lambda": td_lambda, "discounted_return": discounted_return,
          "vtrace": vtrace, "retrace": retrace, "elig_trace": elig_trace,
          "episodic_prefix_sum": episodic_prefix_sum, "affine_scan": affine_scan}[name]
    params = inspect.signature(fn).parameters
    kw = {k: v for k, v in inp.items() if k in params}
    kw.update({k: v for k, v in scal.items() if k in params})
    return fn(**kw)


__all__ = ["gae", "td_lambda", "discounted_return", "vtrace", "retrace", "elig_trace",
           "episodic_prefix_sum", "affine_scan", "affine_scan_grad", "affine_scan_tm", "run"]
