"""GPU parity of the generic affine scan (rlscan_affine_scan) against the
oracle: x_t = b_t + a_t x_prev along T, forward or backward, with resets and
a per-row initial carry.  Same bar as the estimators: |gpu - ref| <= 1e-4 (1 +
|ref|) element by element, on every plan (whole-row blocks of every size,
look-back chains), odd and long rows, unaligned views and host tensors."""
import numpy as np
import pytest
import torch

import oracle
import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build
from segmented_linear_recurrence_b200 import synthetic

from .util import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    slr_build.build()


@pytest.fixture
def options():
    yield slr.rlscan_set_option
    for name, default in (("force_lookback", 0), ("force_block", 0), ("force_scalar", 0)):
        slr.rlscan_set_option(name, default)


def run_both(d, reverse, device="cuda", views=None):
    t = {k: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in d.items()}
    if views is not None:
        t = views(t)
    got = slr.rlscan_affine_scan(t["a"], t["b"], t["reset"], t["init"], reverse=reverse)
    ref = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse)
    return got.cpu().numpy().astype(np.float64), ref


def assert_close(got, ref, what):
    err = np.abs(got - ref)
    bound = TOL * (1.0 + np.abs(ref))
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {bad.shape[0]} elements off, first {tuple(bad[0])}: " \
                          f"gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


CASES = [(512, 128), (64, 2048), (4096, 512), (5, 5000), (40, 96), (33, 1001), (7, 3), (1, 70001), (3, 1)]


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("N,T", CASES)
def test_affine_matches_oracle(N, T, reverse):
    d = synthetic.make_affine_inputs(N, T, seed=2000 + N + T, p_reset=0.01)
    got, ref = run_both(d, reverse)
    assert_close(got, ref, f"N={N} T={T} reverse={reverse}")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("with_reset,with_init", [(False, False), (False, True), (True, False)])
def test_affine_optional_inputs(reverse, with_reset, with_init):
    d = synthetic.make_affine_inputs(96, 777, seed=2101, p_reset=0.02 if with_reset else 0.0,
                                     with_init=with_init)
    got, ref = run_both(d, reverse)
    assert_close(got, ref, f"reset={with_reset} init={with_init}")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("block", [128, 192, 256, 384, 512])
@pytest.mark.parametrize("lookback", [0, 1])
def test_affine_every_plan(reverse, block, lookback, options):
    options("force_block", block)
    options("force_lookback", lookback)
    for N, T in ((100, 100), (3, 9000), (17, 1537)):
        d = synthetic.make_affine_inputs(N, T, seed=2200 + N, p_reset=0.01)
        got, ref = run_both(d, reverse)
        assert_close(got, ref, f"block={block} lookback={lookback} N={N} T={T}")


def test_affine_unit_coefficient_long_row_is_cumsum():
    # a = 1 without resets: the cumulative sum of b over a row of 2^20 steps,
    # a chain of 512 look-back chunks.  b >= 0 so the sums do not cancel: with
    # a = 1 the fp32 error grows with the partial sums, and a zero-mean sum
    # near a crossing of 0 is ill-conditioned for any fp32 evaluation order.
    d = synthetic.make_affine_inputs(2, 1 << 20, seed=2301, p_reset=0.0, with_init=False)
    d["a"][:] = 1.0
    d["b"] = np.abs(d["b"])
    for reverse in (False, True):
        got, ref = run_both(d, reverse)
        assert_close(got, ref, f"cumsum reverse={reverse}")


def test_affine_unaligned_views_and_scalar_path(options):
    d = synthetic.make_affine_inputs(20, 301, seed=2401, p_reset=0.03)

    def shift(t):
        # views starting one element in: no 32-byte alignment anywhere
        out = {}
        for k, v in t.items():
            if v is None:
                out[k] = None
                continue
            big = torch.empty(v.numel() + 1, dtype=v.dtype, device=v.device)
            big[1:] = v.reshape(-1)
            out[k] = big[1:].view(v.shape)
        return out

    for reverse in (False, True):
        got, ref = run_both(d, reverse, views=shift)
        assert_close(got, ref, f"unaligned reverse={reverse}")
    options("force_scalar", 1)
    got, ref = run_both(d, True)
    assert_close(got, ref, "scalar path")


def test_affine_host_tensors():
    d = synthetic.make_affine_inputs(8, 500, seed=2501, p_reset=0.02)
    got, ref = run_both(d, True, device="cpu")
    assert_close(got, ref, "host tensors")


def test_affine_reset_everywhere_returns_b():
    d = synthetic.make_affine_inputs(16, 1000, seed=2601, p_reset=0.0)
    d["reset"] = np.ones_like(d["a"], dtype=np.uint8)
    for reverse in (False, True):
        got, _ = run_both(d, reverse)
        np.testing.assert_array_equal(got, d["b"].astype(np.float64))



# --------------------------------------------------------------------------
# gradient (adjoint) of the affine scan
# --------------------------------------------------------------------------

def run_grad(d, dy, reverse, device="cuda"):
    x_ref = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse).astype(np.float32)
    t = {k: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(device)
         for k, v in dict(d, x=x_ref, dy=dy).items()}
    da, db, dinit = slr.rlscan_affine_scan_grad(t["a"], t["x"], t["dy"], t["reset"], t["init"], reverse=reverse)
    rda, rdb, rdinit = oracle.affine_scan_grad(d["a"], x_ref, dy, d["reset"], d["init"], reverse=reverse)
    return (da.cpu().numpy().astype(np.float64), db.cpu().numpy().astype(np.float64),
            None if dinit is None else dinit.cpu().numpy().astype(np.float64)), (rda, rdb, rdinit)


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("N,T", CASES)
def test_affine_grad_matches_oracle(N, T, reverse):
    d = synthetic.make_affine_inputs(N, T, seed=2700 + N + T, p_reset=0.01)
    dy = np.random.default_rng(N + T).standard_normal((N, T)).astype(np.float32)
    got, ref = run_grad(d, dy, reverse)
    for name, g, r in zip(("da", "db", "dinit"), got, ref):
        assert_close(g, r, f"{name} N={N} T={T} reverse={reverse}")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("block", [128, 256, 512])
@pytest.mark.parametrize("lookback", [0, 1])
def test_affine_grad_every_plan(reverse, block, lookback, options):
    options("force_block", block)
    options("force_lookback", lookback)
    for N, T in ((100, 100), (3, 9000), (17, 1537), (9, 5)):
        d = synthetic.make_affine_inputs(N, T, seed=2800 + N, p_reset=0.02)
        dy = np.random.default_rng(T).standard_normal((N, T)).astype(np.float32)
        got, ref = run_grad(d, dy, reverse)
        for name, g, r in zip(("da", "db", "dinit"), got, ref):
            assert_close(g, r, f"{name} block={block} lookback={lookback} N={N} T={T}")


def test_affine_grad_optional_outputs_and_host_tensors():
    d = synthetic.make_affine_inputs(12, 333, seed=2901, p_reset=0.03, with_init=False)
    dy = np.random.default_rng(7).standard_normal((12, 333)).astype(np.float32)
    x = oracle.affine_scan(d["a"], d["b"], d["reset"], None, reverse=True).astype(np.float32)
    t = {k: torch.from_numpy(v) if v is not None else None for k, v in dict(d, x=x, dy=dy).items()}
    da, db, dinit = slr.rlscan_affine_scan_grad(t["a"], t["x"], t["dy"], t["reset"], None, reverse=True,
                                                need_da=False, need_dinit=False)
    assert da is None and dinit is None
    _, rdb, _ = oracle.affine_scan_grad(d["a"], x, dy, d["reset"], None, reverse=True)
    assert_close(db.numpy().astype(np.float64), rdb, "db only, host tensors")


# --------------------------------------------------------------------------
# bf16 I/O (rlscan_affine_scan_bf16): the oracle runs on the same bf16 values
# widened to fp32 (exact); the result is fp32 arithmetic rounded to bf16 (8
# significant bits: rounding to nearest is off by at most 2^-8 relative), so
# |gpu - ref| <= 2^-8 |ref| + 1.1e-4 (1 + |ref|)
# --------------------------------------------------------------------------

def run_bf16(d, reverse, device="cuda"):
    to16 = lambda v: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).to(torch.bfloat16)  # noqa: E731
    a16, b16, i16 = to16(d["a"]), to16(d["b"]), to16(d["init"])
    rs = None if d["reset"] is None else torch.from_numpy(d["reset"])
    mv = lambda t: None if t is None else t.to(device)  # noqa: E731
    got = slr.rlscan_affine_scan_bf16(mv(a16), mv(b16), mv(rs), mv(i16), reverse=reverse)
    f32 = lambda t: None if t is None else t.float().numpy()  # noqa: E731
    ref = oracle.affine_scan(f32(a16), f32(b16), d["reset"], f32(i16), reverse=reverse)
    return got.float().cpu().numpy().astype(np.float64), ref


def assert_close_bf16(got, ref, what):
    bound = 2.0 ** -8 * np.abs(ref) + 1.1e-4 * (1.0 + np.abs(ref))
    bad = np.argwhere(np.abs(got - ref) > bound)
    assert bad.size == 0, f"{what}: {bad.shape[0]} elements off, first {tuple(bad[0])}: " \
                          f"gpu {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("N,T", CASES)
def test_affine_bf16_matches_oracle(N, T, reverse):
    d = synthetic.make_affine_inputs(N, T, seed=3000 + N + T, p_reset=0.01)
    got, ref = run_bf16(d, reverse)
    assert_close_bf16(got, ref, f"bf16 N={N} T={T} reverse={reverse}")


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("block", [128, 256, 512])
@pytest.mark.parametrize("lookback", [0, 1])
def test_affine_bf16_every_plan(reverse, block, lookback, options):
    options("force_block", block)
    options("force_lookback", lookback)
    for N, T in ((100, 100), (3, 9000), (17, 1537)):
        d = synthetic.make_affine_inputs(N, T, seed=3100 + N, p_reset=0.01)
        got, ref = run_bf16(d, reverse)
        assert_close_bf16(got, ref, f"bf16 block={block} lookback={lookback} N={N} T={T}")


def test_affine_bf16_scalar_path_and_host_tensors(options):
    d = synthetic.make_affine_inputs(11, 333, seed=3201, p_reset=0.02)
    got, ref = run_bf16(d, True, device="cpu")
    assert_close_bf16(got, ref, "bf16 host tensors")
    options("force_scalar", 1)
    got, ref = run_bf16(d, False)
    assert_close_bf16(got, ref, "bf16 scalar path")


# --------------------------------------------------------------------------
# autograd: slr.affine_scan's backward is the adjoint kernel; the gradients
# match the oracle's adjoint of the same forward
# --------------------------------------------------------------------------

@pytest.mark.parametrize("reverse", [False, True])
def test_autograd_affine_scan_matches_oracle_adjoint(reverse):
    N, T = 48, 3000
    d = synthetic.make_affine_inputs(N, T, seed=3400, p_reset=0.01)
    dev = lambda v: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).cuda()  # noqa: E731
    a = dev(d["a"]).requires_grad_()
    b = dev(d["b"]).requires_grad_()
    init = dev(d["init"]).requires_grad_()
    reset = dev(d["reset"])
    rng = np.random.default_rng(3401)
    w = rng.standard_normal((N, T)).astype(np.float32)
    x = slr.affine_scan(a, b, reset, init, reverse=reverse)
    (x * dev(w)).sum().backward()
    xr = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse)
    da, db, di = oracle.affine_scan_grad(d["a"], xr.astype(np.float32), w, d["reset"], d["init"], reverse=reverse)
    for name, got, ref in (("da", a.grad, da), ("db", b.grad, db), ("dinit", init.grad, di)):
        g = got.cpu().numpy().astype(np.float64)
        assert_close(g, ref, f"autograd {name} reverse={reverse}")


def test_autograd_affine_scan_partial_requirements():
    d = synthetic.make_affine_inputs(5, 100, seed=3402, p_reset=0.05)
    a = torch.from_numpy(d["a"]).cuda()
    b = torch.from_numpy(d["b"]).cuda().requires_grad_()
    x = slr.affine_scan(a, b, torch.from_numpy(d["reset"]).cuda(), None)
    x.sum().backward()
    assert b.grad is not None and a.grad is None
    assert torch.isfinite(b.grad).all()
