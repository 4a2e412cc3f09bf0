"""rlscan_gae_noalloc: GAE for callers that cannot allocate device memory.

Some callers must not allocate: code running while its stream is captured
into a CUDA graph, processes whose device memory is owned by another
allocator, latency-critical loops.  rlscan_gae_noalloc keeps its block-to-
block carry scratch in a fixed array inside the library instead.  This test
calls it through the C ABI and checks its output against rlscan_gae's on
the same inputs, for two calls in a row (the second on different data, so
scratch left over from the first call cannot go unnoticed), on rows long
enough to use the scratch and on rows that fit one block.  It runs last
(file order) and needs nothing from the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build
from segmented_linear_recurrence_b200 import synthetic

from .util import TOL, assert_parity

pytestmark = pytest.mark.gpu

VP, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float


def _noalloc_fn():
    fn = slr.lib().rlscan_gae_noalloc
    fn.argtypes = [VP] * 8 + [I64, I64, F, F, VP]
    fn.restype = ctypes.c_int
    return fn


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("N,T", [(3, 50_000), (16, 3_000), (512, 128)])
def test_noalloc_gae_matches_gae_on_two_calls(N, T):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()
    fn = _noalloc_fn()
    gamma, lam = float(np.float32(0.99)), float(np.float32(0.95))
    stream = torch.cuda.current_stream()
    for call, seed in enumerate((901, 902)):
        d = synthetic.make_inputs("gae", N, T, seed=seed + N, p_term=0.002, p_trunc=0.002)
        t = {k: (None if v is None else torch.from_numpy(v).cuda()) for k, v in d.items()}
        ref_adv, ref_ret = slr.rlscan_gae(t["rewards"], t["values"], t["bootstrap"], t["terminated"],
                                          t["truncated"], t["trunc_value"], gamma=gamma, lam=lam)
        adv = torch.full((N, T), float("nan"), device="cuda")
        ret = torch.full((N, T), float("nan"), device="cuda")
        st = fn(_ptr(t["rewards"]), _ptr(t["values"]), _ptr(t["bootstrap"]), _ptr(t["terminated"]),
                _ptr(t["truncated"]), _ptr(t["trunc_value"]), _ptr(adv), _ptr(ret), N, T, gamma, lam,
                ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, slr.STATUS.get(st, st)
        assert slr.rlscan_sync_status() == 0
        assert_parity("gae", (adv.cpu().numpy(), ret.cpu().numpy()),
                      (ref_adv.cpu().numpy(), ref_ret.cpu().numpy()), tol=TOL, what=f"call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fn = _noalloc_fn()
    base = 0x7F0000000000  # never dereferenced: the size check comes first
    p = [ctypes.c_void_p(base + i * (1 << 34)) for i in range(8)]
    st = fn(p[0], p[1], p[2], None, None, None, p[3], p[4], 1 << 14, (1 << 13) + 1, 0.99, 0.95, None)
    assert slr.STATUS[st] == "RLSCAN_ERR_TOO_LARGE"
