"""Python binding of librlscan: torch tensors in, the C ABI of ``include/rlscan.h`` underneath.

Every function here only marshals arguments: it checks dtypes and shapes,
allocates missing outputs with torch, passes raw device pointers and the
current CUDA stream to the same-named ``extern "C"`` entry point, and turns a
non-OK status into :class:`RlscanError`.  All arithmetic runs in the CUDA
kernels of ``librlscan.so``; there is no CPU fallback -- if the library is
missing or no GPU is present, the call raises.

Host (CPU) tensors are accepted too: they are copied to the current CUDA
device on the current stream, the kernel runs there, and the outputs are
copied back into (pinned, when the inputs were pinned) host tensors.  Use
pinned inputs for asynchronous copies.
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

__all__ = [
    "RlscanError", "lib", "rlscan_gae", "rlscan_vtrace", "rlscan_retrace", "rlscan_td_lambda",
    "rlscan_discounted_return", "rlscan_elig_trace", "rlscan_episodic_prefix_sum",
    "rlscan_affine_scan", "rlscan_affine_scan_grad", "rlscan_affine_scan_bf16", "rlscan_sync_status", "rlscan_status_string", "rlscan_release_workspaces",
    "rlscan_abi_version", "rlscan_query_plan", "rlscan_set_option", "rlscan_get_option",
    "rlscan_reserve_workspace", "rlscan_gae_tm", "rlscan_vtrace_tm", "rlscan_td_lambda_tm",
    "rlscan_discounted_return_tm", "rlscan_elig_trace_tm", "rlscan_episodic_prefix_sum_tm",
    "rlscan_affine_scan_tm", "rlscan_query_plan_tm", "rlscan_gae_bf16", "affine_scan",
    "STATUS", "OPTIONS", "ESTIMATOR_IDS", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librlscan.so")

STATUS = {0: "RLSCAN_OK", 1: "RLSCAN_ERR_INVALID_ARG", 2: "RLSCAN_ERR_OVERLAP",
          3: "RLSCAN_ERR_LAUNCH", 4: "RLSCAN_ERR_TIMEOUT", 5: "RLSCAN_ERR_NOMEM",
          6: "RLSCAN_ERR_CUDA", 7: "RLSCAN_ERR_CAPTURE", 8: "RLSCAN_ERR_TOO_LARGE"}
OPTIONS = {"lookback_timeout_ns": 1, "force_lookback": 2, "force_block": 3, "force_scalar": 4,
           "check_pointers": 5, "test_starve_lookback": 6, "pdl": 7}
ESTIMATOR_IDS = {"gae": 0, "vtrace": 1, "retrace": 2, "td_lambda": 3, "discounted_return": 4,
                 "elig_trace": 5, "episodic_prefix_sum": 6, "affine_scan": 7, "affine_scan_grad": 8,
                 "affine_scan_bf16": 9, "gae_bf16": 10}


class RlscanError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = int(status)
        super().__init__(f"{fn} failed: {STATUS.get(self.status, self.status)}")


class PlanInfo(ctypes.Structure):
    _fields_ = [("block_threads", ctypes.c_int32), ("chunk_steps", ctypes.c_int32),
                ("lookback", ctypes.c_int32), ("launches", ctypes.c_int32),
                ("chunks", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


_lib = None
_VP, _I64, _F, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int
_SIGNATURES = {
    "rlscan_gae": [_VP] * 8 + [_I64, _I64, _F, _F, _VP],
    "rlscan_vtrace": [_VP] * 9 + [_I64, _I64, _F, _F, _F, _F, _VP],
    "rlscan_retrace": [_VP] * 10 + [_I64, _I64, _I64, _F, _F, _VP],
    "rlscan_td_lambda": [_VP] * 7 + [_I64, _I64, _F, _F, _VP],
    "rlscan_discounted_return": [_VP] * 6 + [_I64, _I64, _F, _VP],
    "rlscan_elig_trace": [_VP] * 5 + [_I64, _I64, _F, _F, _VP],
    "rlscan_episodic_prefix_sum": [_VP] * 4 + [_I64, _I64, _VP],
    "rlscan_affine_scan": [_VP] * 5 + [_I64, _I64, ctypes.c_int32, _VP],
    "rlscan_affine_scan_grad": [_VP] * 8 + [_I64, _I64, ctypes.c_int32, _VP],
    "rlscan_affine_scan_bf16": [_VP] * 5 + [_I64, _I64, ctypes.c_int32, _VP],
    "rlscan_gae_bf16": [_VP] * 8 + [_I64, _I64, _F, _F, _VP],
    "rlscan_gae_tm": [_VP] * 8 + [_I64, _I64, _F, _F, _VP],
    "rlscan_vtrace_tm": [_VP] * 9 + [_I64, _I64, _F, _F, _F, _F, _VP],
    "rlscan_td_lambda_tm": [_VP] * 7 + [_I64, _I64, _F, _F, _VP],
    "rlscan_discounted_return_tm": [_VP] * 6 + [_I64, _I64, _F, _VP],
    "rlscan_elig_trace_tm": [_VP] * 5 + [_I64, _I64, _F, _F, _VP],
    "rlscan_episodic_prefix_sum_tm": [_VP] * 4 + [_I64, _I64, _VP],
    "rlscan_affine_scan_tm": [_VP] * 5 + [_I64, _I64, ctypes.c_int32, _VP],
    "rlscan_query_plan_tm": [_I, _I64, _I64, ctypes.POINTER(PlanInfo)],
    "rlscan_sync_status": [_VP],
    "rlscan_release_workspaces": [],
    "rlscan_reserve_workspace": [_I64, _VP],
    "rlscan_abi_version": [],
    "rlscan_query_plan": [_I, _I64, _I64, _I64, ctypes.POINTER(PlanInfo)],
    "rlscan_set_option": [_I, _I64],
    "rlscan_get_option": [_I],
    "rlscan_status_string": [_I],
}


def lib():
    """The loaded librlscan (ctypes), with argument types declared.

    Raises RuntimeError if the shared library has not been built: there is
    no other implementation to fall back to."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"librlscan.so is missing ({LIB_PATH}); build it with "
                               "`python -m segmented_linear_recurrence_b200.build`")
        cdll = ctypes.CDLL(LIB_PATH)
        for name, argtypes in _SIGNATURES.items():
            fn = getattr(cdll, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_int
        cdll.rlscan_status_string.restype = ctypes.c_char_p
        cdll.rlscan_get_option.restype = ctypes.c_int64
        cdll.rlscan_release_workspaces.restype = None
        _lib = cdll
    return _lib


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

class _Call:
    """Collects the device tensors of one call; moves host tensors to the GPU."""

    def __init__(self, name, ref):
        self.name = name
        if ref.is_cuda:
            self.device = ref.device
            self.host = False
        else:
            if not torch.cuda.is_available():
                raise RuntimeError(f"{name}: librlscan needs a CUDA device")
            self.device = torch.device("cuda", torch.cuda.current_device())
            self.host = True
            self.pinned = ref.is_pinned()
        self.keep = []

    def tensor(self, x, dtype, shape, what, required=True):
        if x is None:
            if required:
                raise ValueError(f"{self.name}: {what} is required")
            return None
        if not isinstance(x, torch.Tensor):
            raise TypeError(f"{self.name}: {what} must be a torch.Tensor")
        if x.dtype != dtype and not (dtype == torch.uint8 and x.dtype == torch.bool):
            raise TypeError(f"{self.name}: {what} must be {dtype}, got {x.dtype}")
        if tuple(x.shape) != tuple(shape):
            raise ValueError(f"{self.name}: {what} must have shape {tuple(shape)}, got {tuple(x.shape)}")
        if self.host:
            if x.is_cuda:
                raise ValueError(f"{self.name}: mix of host and device tensors")
            x = x.to(self.device, non_blocking=True)
        elif x.device != self.device:
            raise ValueError(f"{self.name}: {what} is on {x.device}, expected {self.device}")
        if not x.is_contiguous():
            raise ValueError(f"{self.name}: {what} must be contiguous")
        self.keep.append(x)
        return x

    def output(self, x, dtype, shape, what):
        if x is None:
            x = torch.empty(shape, dtype=dtype, device=self.device)
        elif self.host:
            raise ValueError(f"{self.name}: pass no {what} buffer when the inputs are host tensors")
        else:
            self.tensor(x, dtype, shape, what)
        self.keep.append(x)
        return x

    @staticmethod
    def ptr(x):
        return None if x is None else ctypes.c_void_p(x.data_ptr())

    def stream(self, stream):
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        return ctypes.c_void_p(s.cuda_stream)

    def finish(self, status, outs):
        if status != 0:
            raise RlscanError(self.name, status)
        if not self.host:
            return outs
        res = []
        for o in outs:
            if o is None:
                res.append(None)
                continue
            h = torch.empty(o.shape, dtype=o.dtype, pin_memory=self.pinned)
            h.copy_(o, non_blocking=self.pinned)
            res.append(h)
        if self.pinned:
            torch.cuda.current_stream(self.device).synchronize()
        return tuple(res)


def _nt(x, name, tm=False):
    """(N, T) of a per-step tensor: [N, T] row-major, or [T, N] time-major."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name}: per-step inputs must be 2-D {'[T, N]' if tm else '[N, T]'} tensors")
    return (int(x.shape[1]), int(x.shape[0])) if tm else (int(x.shape[0]), int(x.shape[1]))


def _layout_dispatch(fn):
    """Per-step tensors given as [N, T] views of time-major [T, N] storage
    (every 2-D argument non-contiguous with a contiguous transpose, as
    `buf.T` gives) run on the time-major kernel without a copy; the outputs
    come back as [N, T] views of time-major buffers."""
    def is2d(x):
        return isinstance(x, torch.Tensor) and x.dim() == 2

    @functools.wraps(fn)
    def wrapper(*args, **kw):
        if kw.get("_tm"):
            return fn(*args, **kw)
        mats = [x for x in list(args) + list(kw.values()) if is2d(x)]
        if mats and all(not x.is_contiguous() and x.t().is_contiguous() for x in mats):
            res = fn(*[x.t() if is2d(x) else x for x in args], _tm=True,
                     **{k: (v.t() if is2d(v) else v) for k, v in kw.items()})
            if isinstance(res, tuple):
                return tuple(None if r is None else r.t() for r in res)
            return res.t()
        return fn(*args, **kw)
    return wrapper


# ---------------------------------------------------------------------------
# estimators
# ---------------------------------------------------------------------------

@_layout_dispatch
def rlscan_gae(rewards, values, bootstrap, terminated=None, truncated=None, trunc_value=None, *,
               gamma=0.99, lam=0.95, advantages=None, returns=None, want_returns=True, stream=None, _tm=False):
    """GAE advantages and returns.  Returns (advantages, returns or None)."""
    name = "rlscan_gae_tm" if _tm else "rlscan_gae"
    N, T = _nt(rewards, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, rewards)
    r = c.tensor(rewards, torch.float32, S, "rewards")
    v = c.tensor(values, torch.float32, S, "values")
    b = c.tensor(bootstrap, torch.float32, (N,), "bootstrap")
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    tv = c.tensor(trunc_value, torch.float32, S, "trunc_value", required=tr is not None)
    adv = c.output(advantages, torch.float32, S, "advantages")
    ret = c.output(returns, torch.float32, S, "returns") if (want_returns or returns is not None) else None
    st = getattr(lib(), name)(c.ptr(r), c.ptr(v), c.ptr(b), c.ptr(te), c.ptr(tr), c.ptr(tv), c.ptr(adv),
                          c.ptr(ret), N, T, float(gamma), float(lam), c.stream(stream))
    return c.finish(st, (adv, ret))


@_layout_dispatch
def rlscan_vtrace(log_rhos, rewards, values, bootstrap, terminated=None, truncated=None,
                  trunc_value=None, *, gamma=0.99, lam=1.0, rho_bar=1.0, c_bar=1.0, vs=None,
                  pg_advantages=None, want_pg=True, stream=None, _tm=False):
    """V-trace targets vs and policy-gradient advantages.  Returns (vs, pg or None)."""
    name = "rlscan_vtrace_tm" if _tm else "rlscan_vtrace"
    N, T = _nt(rewards, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, rewards)
    lr = c.tensor(log_rhos, torch.float32, S, "log_rhos")
    r = c.tensor(rewards, torch.float32, S, "rewards")
    v = c.tensor(values, torch.float32, S, "values")
    b = c.tensor(bootstrap, torch.float32, (N,), "bootstrap")
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    tv = c.tensor(trunc_value, torch.float32, S, "trunc_value", required=tr is not None)
    out_vs = c.output(vs, torch.float32, S, "vs")
    pg = c.output(pg_advantages, torch.float32, S, "pg_advantages") if (want_pg or pg_advantages is not None) else None
    st = getattr(lib(), name)(c.ptr(lr), c.ptr(r), c.ptr(v), c.ptr(b), c.ptr(te), c.ptr(tr), c.ptr(tv),
                             c.ptr(out_vs), c.ptr(pg), N, T, float(gamma), float(lam),
                             float(rho_bar), float(c_bar), c.stream(stream))
    return c.finish(st, (out_vs, pg))


def rlscan_retrace(q, pi, mu_a, actions, rewards, bootstrap, terminated=None, truncated=None,
                   trunc_value=None, *, gamma=0.99, lam=0.95, q_ret=None, stream=None):
    """Retrace(lambda) targets for the taken actions.  Returns q_ret."""
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise ValueError("rlscan_retrace: q must be a 3-D [N, T, A] tensor")
    N, T, A = (int(s) for s in q.shape)
    c = _Call("rlscan_retrace", q)
    qq = c.tensor(q, torch.float32, (N, T, A), "q")
    pp = c.tensor(pi, torch.float32, (N, T, A), "pi")
    mu = c.tensor(mu_a, torch.float32, (N, T), "mu_a")
    ac = c.tensor(actions, torch.int32, (N, T), "actions")
    r = c.tensor(rewards, torch.float32, (N, T), "rewards")
    b = c.tensor(bootstrap, torch.float32, (N,), "bootstrap")
    te = c.tensor(terminated, torch.uint8, (N, T), "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, (N, T), "truncated", required=False)
    tv = c.tensor(trunc_value, torch.float32, (N, T), "trunc_value", required=tr is not None)
    out = c.output(q_ret, torch.float32, (N, T), "q_ret")
    st = lib().rlscan_retrace(c.ptr(qq), c.ptr(pp), c.ptr(mu), c.ptr(ac), c.ptr(r), c.ptr(b), c.ptr(te),
                              c.ptr(tr), c.ptr(tv), c.ptr(out), N, T, A, float(gamma), float(lam),
                              c.stream(stream))
    return c.finish(st, (out,))[0]


@_layout_dispatch
def rlscan_td_lambda(rewards, values, bootstrap, terminated=None, truncated=None, trunc_value=None,
                     *, gamma=0.99, lam=0.95, returns=None, stream=None, _tm=False):
    """TD(lambda) returns.  Returns the [N, T] returns."""
    name = "rlscan_td_lambda_tm" if _tm else "rlscan_td_lambda"
    N, T = _nt(rewards, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, rewards)
    r = c.tensor(rewards, torch.float32, S, "rewards")
    v = c.tensor(values, torch.float32, S, "values")
    b = c.tensor(bootstrap, torch.float32, (N,), "bootstrap")
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    tv = c.tensor(trunc_value, torch.float32, S, "trunc_value", required=tr is not None)
    out = c.output(returns, torch.float32, S, "returns")
    st = getattr(lib(), name)(c.ptr(r), c.ptr(v), c.ptr(b), c.ptr(te), c.ptr(tr), c.ptr(tv), c.ptr(out),
                                N, T, float(gamma), float(lam), c.stream(stream))
    return c.finish(st, (out,))[0]


@_layout_dispatch
def rlscan_discounted_return(rewards, bootstrap=None, terminated=None, truncated=None,
                             trunc_value=None, *, gamma=0.99, returns=None, stream=None, _tm=False):
    """Discounted returns (bootstrap optional).  Returns the [N, T] returns."""
    name = "rlscan_discounted_return_tm" if _tm else "rlscan_discounted_return"
    N, T = _nt(rewards, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, rewards)
    r = c.tensor(rewards, torch.float32, S, "rewards")
    b = c.tensor(bootstrap, torch.float32, (N,), "bootstrap", required=False)
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    tv = c.tensor(trunc_value, torch.float32, S, "trunc_value", required=tr is not None)
    out = c.output(returns, torch.float32, S, "returns")
    st = getattr(lib(), name)(c.ptr(r), c.ptr(b), c.ptr(te), c.ptr(tr), c.ptr(tv), c.ptr(out),
                                        N, T, float(gamma), c.stream(stream))
    return c.finish(st, (out,))[0]


@_layout_dispatch
def rlscan_elig_trace(inputs, init_trace=None, terminated=None, truncated=None, *, gamma=0.99,
                      lam=0.95, traces=None, stream=None, _tm=False):
    """Accumulating eligibility traces (forward in time).  Returns the [N, T] traces."""
    name = "rlscan_elig_trace_tm" if _tm else "rlscan_elig_trace"
    N, T = _nt(inputs, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, inputs)
    g = c.tensor(inputs, torch.float32, S, "inputs")
    e0 = c.tensor(init_trace, torch.float32, (N,), "init_trace", required=False)
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    out = c.output(traces, torch.float32, S, "traces")
    st = getattr(lib(), name)(c.ptr(g), c.ptr(e0), c.ptr(te), c.ptr(tr), c.ptr(out), N, T,
                                 float(gamma), float(lam), c.stream(stream))
    return c.finish(st, (out,))[0]


@_layout_dispatch
def rlscan_episodic_prefix_sum(x, terminated=None, truncated=None, *, out=None, stream=None, _tm=False):
    """Episodic inclusive prefix sums of int32 values.  Returns the [N, T] int32 sums."""
    name = "rlscan_episodic_prefix_sum_tm" if _tm else "rlscan_episodic_prefix_sum"
    N, T = _nt(x, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, x)
    xx = c.tensor(x, torch.int32, S, "x")
    te = c.tensor(terminated, torch.uint8, S, "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, S, "truncated", required=False)
    o = c.output(out, torch.int32, S, "out")
    st = getattr(lib(), name)(c.ptr(xx), c.ptr(te), c.ptr(tr), c.ptr(o), N, T,
                                          c.stream(stream))
    return c.finish(st, (o,))[0]


@_layout_dispatch
def rlscan_affine_scan(a, b, reset=None, init=None, *, reverse=False, x=None, stream=None, _tm=False):
    """Generic affine scan x_t = b_t + a_t x_prev along T (backward when
    `reverse`), x_prev = init[n] at the row's first step, x_t = b_t where
    reset.  Returns the [N, T] float32 x."""
    name = "rlscan_affine_scan_tm" if _tm else "rlscan_affine_scan"
    N, T = _nt(a, name, _tm)
    S = (T, N) if _tm else (N, T)
    c = _Call(name, a)
    aa = c.tensor(a, torch.float32, S, "a")
    bb = c.tensor(b, torch.float32, S, "b")
    rs = c.tensor(reset, torch.uint8, S, "reset", required=False)
    x0 = c.tensor(init, torch.float32, (N,), "init", required=False)
    out = c.output(x, torch.float32, S, "x")
    st = getattr(lib(), name)(c.ptr(aa), c.ptr(bb), c.ptr(rs), c.ptr(x0), c.ptr(out), N, T,
                                  1 if reverse else 0, c.stream(stream))
    return c.finish(st, (out,))[0]


def rlscan_gae_bf16(rewards, values, bootstrap, terminated=None, truncated=None, trunc_value=None, *,
                    gamma=0.99, lam=0.95, advantages=None, returns=None, want_returns=True, stream=None):
    """rlscan_gae on bfloat16 tensors (fp32 arithmetic, bf16 results).
    Returns (advantages, returns or None)."""
    N, T = _nt(rewards, "rlscan_gae_bf16")
    c = _Call("rlscan_gae_bf16", rewards)
    r = c.tensor(rewards, torch.bfloat16, (N, T), "rewards")
    v = c.tensor(values, torch.bfloat16, (N, T), "values")
    b = c.tensor(bootstrap, torch.bfloat16, (N,), "bootstrap")
    te = c.tensor(terminated, torch.uint8, (N, T), "terminated", required=False)
    tr = c.tensor(truncated, torch.uint8, (N, T), "truncated", required=False)
    tv = c.tensor(trunc_value, torch.bfloat16, (N, T), "trunc_value", required=tr is not None)
    adv = c.output(advantages, torch.bfloat16, (N, T), "advantages")
    ret = c.output(returns, torch.bfloat16, (N, T), "returns") if (want_returns or returns is not None) else None
    st = lib().rlscan_gae_bf16(c.ptr(r), c.ptr(v), c.ptr(b), c.ptr(te), c.ptr(tr), c.ptr(tv), c.ptr(adv),
                               c.ptr(ret), N, T, float(gamma), float(lam), c.stream(stream))
    return c.finish(st, (adv, ret))


def rlscan_affine_scan_bf16(a, b, reset=None, init=None, *, reverse=False, x=None, stream=None):
    """rlscan_affine_scan on bfloat16 tensors (fp32 arithmetic, bf16 result).
    Returns the [N, T] bfloat16 x."""
    N, T = _nt(a, "rlscan_affine_scan_bf16")
    c = _Call("rlscan_affine_scan_bf16", a)
    aa = c.tensor(a, torch.bfloat16, (N, T), "a")
    bb = c.tensor(b, torch.bfloat16, (N, T), "b")
    rs = c.tensor(reset, torch.uint8, (N, T), "reset", required=False)
    x0 = c.tensor(init, torch.bfloat16, (N,), "init", required=False)
    out = c.output(x, torch.bfloat16, (N, T), "x")
    st = lib().rlscan_affine_scan_bf16(c.ptr(aa), c.ptr(bb), c.ptr(rs), c.ptr(x0), c.ptr(out), N, T,
                                       1 if reverse else 0, c.stream(stream))
    return c.finish(st, (out,))[0]


def rlscan_affine_scan_grad(a, x, dy, reset=None, init=None, *, reverse=False, need_da=True,
                            need_dinit=True, da=None, db=None, dinit=None, stream=None):
    """Gradient of rlscan_affine_scan given the forward output `x` and the
    upstream gradient `dy`.  Returns (da, db, dinit); da / dinit are None
    when not requested."""
    N, T = _nt(a, "rlscan_affine_scan_grad")
    c = _Call("rlscan_affine_scan_grad", a)
    aa = c.tensor(a, torch.float32, (N, T), "a")
    xx = c.tensor(x, torch.float32, (N, T), "x")
    gy = c.tensor(dy, torch.float32, (N, T), "dy")
    rs = c.tensor(reset, torch.uint8, (N, T), "reset", required=False)
    x0 = c.tensor(init, torch.float32, (N,), "init", required=False)
    o_db = c.output(db, torch.float32, (N, T), "db")
    o_da = c.output(da, torch.float32, (N, T), "da") if (need_da or da is not None) else None
    o_di = c.output(dinit, torch.float32, (N,), "dinit") if (need_dinit or dinit is not None) else None
    st = lib().rlscan_affine_scan_grad(c.ptr(aa), c.ptr(xx), c.ptr(gy), c.ptr(rs), c.ptr(x0), c.ptr(o_da),
                                       c.ptr(o_db), c.ptr(o_di), N, T, 1 if reverse else 0, c.stream(stream))
    return c.finish(st, (o_da, o_db, o_di))


class _AffineScanFn(torch.autograd.Function):
    """Autograd glue: the forward is rlscan_affine_scan, the backward its adjoint
    kernel rlscan_affine_scan_grad (nothing is computed here)."""

    @staticmethod
    def forward(ctx, a, b, init, reset, reverse):
        x = rlscan_affine_scan(a, b, reset, init, reverse=reverse)
        ctx.save_for_backward(a, x, init)
        ctx.reset, ctx.reverse = reset, reverse
        return x

    @staticmethod
    def backward(ctx, dy):
        a, x, init = ctx.saved_tensors
        need_da, need_db, need_di = ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2]
        if not (need_da or need_db or need_di):
            return None, None, None, None, None
        da, db, di = rlscan_affine_scan_grad(a, x, dy.contiguous(), ctx.reset, init, reverse=ctx.reverse,
                                             need_da=need_da, need_dinit=need_di and init is not None)
        return (da if need_da else None, db if need_db else None, di if need_di else None, None, None)


def affine_scan(a, b, reset=None, init=None, *, reverse=False):
    """Differentiable rlscan_affine_scan for torch autograd: gradients with
    respect to a, b and init come from the adjoint scan kernel."""
    return _AffineScanFn.apply(a, b, init, reset, bool(reverse))


# ---------------------------------------------------------------------------
# status, options, plans
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# time-major [T, N] variants: same arguments and results, every per-step
# tensor [T, N] (per-environment tensors stay [N])
# ---------------------------------------------------------------------------

def rlscan_gae_tm(*args, **kw):
    """rlscan_gae on time-major [T, N] tensors.  Returns (advantages, returns or None)."""
    return rlscan_gae(*args, _tm=True, **kw)


def rlscan_vtrace_tm(*args, **kw):
    """rlscan_vtrace on time-major [T, N] tensors.  Returns (vs, pg or None)."""
    return rlscan_vtrace(*args, _tm=True, **kw)


def rlscan_td_lambda_tm(*args, **kw):
    """rlscan_td_lambda on time-major [T, N] tensors."""
    return rlscan_td_lambda(*args, _tm=True, **kw)


def rlscan_discounted_return_tm(*args, **kw):
    """rlscan_discounted_return on time-major [T, N] tensors."""
    return rlscan_discounted_return(*args, _tm=True, **kw)


def rlscan_elig_trace_tm(*args, **kw):
    """rlscan_elig_trace on time-major [T, N] tensors."""
    return rlscan_elig_trace(*args, _tm=True, **kw)


def rlscan_episodic_prefix_sum_tm(*args, **kw):
    """rlscan_episodic_prefix_sum on time-major [T, N] tensors."""
    return rlscan_episodic_prefix_sum(*args, _tm=True, **kw)


def rlscan_affine_scan_tm(*args, **kw):
    """rlscan_affine_scan on time-major [T, N] tensors."""
    return rlscan_affine_scan(*args, _tm=True, **kw)


def rlscan_sync_status(stream=None, raise_on_error=False):
    """Synchronize the stream and return (and clear) the device-side status code."""
    s = torch.cuda.current_stream() if stream is None else stream
    st = int(lib().rlscan_sync_status(ctypes.c_void_p(s.cuda_stream)))
    if raise_on_error and st != 0:
        raise RlscanError("rlscan_sync_status", st)
    return st


def rlscan_status_string(status: int) -> str:
    return lib().rlscan_status_string(int(status)).decode()


def rlscan_release_workspaces():
    lib().rlscan_release_workspaces()


def rlscan_reserve_workspace(nbytes: int, stream=None):
    """Allocate the (device, stream) workspace now, e.g. before graph capture."""
    s = torch.cuda.current_stream() if stream is None else stream
    st = lib().rlscan_reserve_workspace(int(nbytes), ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise RlscanError("rlscan_reserve_workspace", st)


def rlscan_abi_version() -> int:
    return int(lib().rlscan_abi_version())


def rlscan_query_plan(estimator: str, N: int, T: int, A: int = 1) -> dict:
    info = PlanInfo()
    st = lib().rlscan_query_plan(ESTIMATOR_IDS[estimator], int(N), int(T), int(A), ctypes.byref(info))
    if st != 0:
        raise RlscanError("rlscan_query_plan", st)
    return {f: getattr(info, f) for f, _ in PlanInfo._fields_}


def rlscan_query_plan_tm(estimator: str, N: int, T: int) -> dict:
    info = PlanInfo()
    st = lib().rlscan_query_plan_tm(ESTIMATOR_IDS[estimator], int(N), int(T), ctypes.byref(info))
    if st != 0:
        raise RlscanError("rlscan_query_plan_tm", st)
    return {f: getattr(info, f) for f, _ in PlanInfo._fields_}


def rlscan_set_option(name: str, value: int):
    st = lib().rlscan_set_option(OPTIONS[name], int(value))
    if st != 0:
        raise RlscanError("rlscan_set_option", st)


def rlscan_get_option(name: str) -> int:
    return int(lib().rlscan_get_option(OPTIONS[name]))
