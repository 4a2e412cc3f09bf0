"""GPU parity of GAE with bfloat16 I/O (rlscan_gae_bf16) against the oracle.

The oracle runs on the same bf16 values widened to fp32 (exact).  The kernel
computes in fp32 and rounds each output to bf16 (8 significant bits: rounding
to nearest is off by at most 2^-8 relative), so the bound is
|gpu - ref| <= 2^-8 |ref| + 1.1e-4 (1 + |ref|): one output rounding on top of
the fp32 bar.  Covers every plan (whole-row blocks of every size, look-back
chains), truncation with bf16 trunc_value, the scalar path and host tensors."""
import numpy as np
import pytest
import torch

import oracle
import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build
from segmented_linear_recurrence_b200 import synthetic

pytestmark = pytest.mark.gpu

REALS = ("rewards", "values", "bootstrap", "trunc_value")


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


def run(d, device="cuda", want_returns=True):
    """bf16 GAE on the bf16-rounded inputs, and the oracle on the same values."""
    t16 = {k: None if d.get(k) is None else torch.from_numpy(np.ascontiguousarray(d[k])).to(torch.bfloat16)
           for k in REALS}
    flags = {k: None if d.get(k) is None else torch.from_numpy(d[k]) for k in ("terminated", "truncated")}
    mv = lambda t: None if t is None else t.to(device)  # noqa: E731
    s = {k: float(np.float32(v)) for k, v in synthetic.SCALARS["gae"].items()}
    adv, ret = slr.rlscan_gae_bf16(mv(t16["rewards"]), mv(t16["values"]), mv(t16["bootstrap"]),
                                   mv(flags["terminated"]), mv(flags["truncated"]), mv(t16["trunc_value"]),
                                   want_returns=want_returns, **s)
    wide = dict(d)
    for k in REALS:
        wide[k] = None if t16[k] is None else t16[k].float().numpy()
    ref = oracle.run("gae", wide, **s)
    got = (adv.float().cpu().numpy().astype(np.float64), None if ret is None else ret.float().cpu().numpy())
    return got, ref


def assert_close(got, ref, what):
    for name, g, r in zip(("advantages", "returns"), got, ref):
        if g is None:
            continue
        bound = 2.0 ** -8 * np.abs(r) + 1.1e-4 * (1.0 + np.abs(r))
        bad = np.argwhere(np.abs(g - r) > bound)
        assert bad.size == 0, f"{what} {name}: {bad.shape[0]} off, first {tuple(bad[0])}: gpu {g[tuple(bad[0])]} " \
                              f"ref {r[tuple(bad[0])]}"


CASES = [(4096, 512), (64, 2048), (512, 128), (5, 5000), (40, 96), (33, 1001), (7, 3), (1, 70001)]


@pytest.mark.parametrize("N,T", CASES)
def test_gae_bf16_matches_oracle(N, T):
    d = synthetic.make_inputs("gae", N, T, seed=5000 + N + T, p_term=0.01, p_trunc=0.01)
    got, ref = run(d)
    assert_close(got, ref, f"N={N} T={T}")


@pytest.mark.parametrize("block", [128, 256, 512])
@pytest.mark.parametrize("lookback", [0, 1])
def test_gae_bf16_every_plan(block, lookback, options):
    options("force_block", block)
    options("force_lookback", lookback)
    for N, T in ((100, 100), (3, 9000), (17, 1537)):
        d = synthetic.make_inputs("gae", N, T, seed=5100 + N, p_term=0.02, p_trunc=0.02)
        got, ref = run(d)
        assert_close(got, ref, f"block={block} lookback={lookback} N={N} T={T}")


def test_gae_bf16_scalar_path_host_tensors_no_returns(options):
    d = synthetic.make_inputs("gae", 11, 333, seed=5201, p_term=0.02, p_trunc=0.02)
    got, ref = run(d, device="cpu")
    assert_close(got, ref, "host tensors")
    options("force_scalar", 1)
    got, ref = run(d, want_returns=False)
    assert got[1] is None
    assert_close(got, ref, "scalar path")


def test_gae_bf16_rounds_like_the_fp32_call():
    # The bf16 call equals the fp32 call on the widened inputs, rounded once.
    d = synthetic.make_inputs("gae", 256, 700, seed=5300, p_term=0.01, p_trunc=0.01)
    t16 = {k: None if d.get(k) is None else torch.from_numpy(d[k]).to(torch.bfloat16).cuda() for k in REALS}
    te = torch.from_numpy(d["terminated"]).cuda()
    tr = torch.from_numpy(d["truncated"]).cuda()
    s = {k: float(np.float32(v)) for k, v in synthetic.SCALARS["gae"].items()}
    a16, r16 = slr.rlscan_gae_bf16(t16["rewards"], t16["values"], t16["bootstrap"], te, tr, t16["trunc_value"], **s)
    a32, r32 = slr.rlscan_gae(t16["rewards"].float(), t16["values"].float(), t16["bootstrap"].float(), te, tr,
                              t16["trunc_value"].float(), **s)
    # same fp32 arithmetic in both kernels (same plan, same order): bit-equal after rounding
    assert torch.equal(a16, a32.to(torch.bfloat16))
    assert torch.equal(r16, r32.to(torch.bfloat16))
