"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

The rl-triton pages print no worked example, so the oracle is pinned by:
  * closed forms (geometric sums) for constant inputs;
  * brute-force, NON-recursive definitions of each estimator (n-step /
    lambda-weighted sums, the IMPALA and Munos et al. off-policy sums, the
    per-episode trace and prefix sums), evaluated on exhaustive flag patterns
    of short rows -- written here from the estimators' original papers, not
    from the oracle's recursions;
  * cross-estimator identities and special cases (gamma = 0, lambda in {0, 1},
    on-policy ratios, one-hot target policies);
  * episode isolation: an input change inside one episode leaves every output
    of the other episodes bit-identical.
A plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a boundary rule applied on the wrong step) breaks at
least one of these.
"""
import itertools

import numpy as np
import pytest

import oracle
from segmented_linear_recurrence_b200 import synthetic

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

G, L = 0.9, 0.8  # generic scalars for the pins (not fp32-rounded: all fp64)


# --------------------------------------------------------------------------
# brute-force definitions (non-recursive), one row at a time
# --------------------------------------------------------------------------

def _boundary(t, T, term, trunc):
    """First step K >= t whose transition does not continue inside the window."""
    k = t
    while True:
        if term[k] or (trunc is not None and trunc[k]) or k == T - 1:
            return k
        k += 1


def _nv(K, n, term, trunc, tv, boot):
    if term[K]:
        return 0.0
    if trunc is not None and trunc[K]:
        return float(tv[K])
    return 0.0 if boot is None else float(boot[n])


def bf_gae(r, v, boot, term, trunc, tv, g, lam):
    N, T = r.shape
    out = np.zeros((N, T))
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            s = 0.0
            for k in range(t, K + 1):
                succ = float(v[n, k + 1]) if k < K else nvK
                delta = float(r[n, k]) + g * succ - float(v[n, k])
                s += (g * lam) ** (k - t) * delta
            out[n, t] = s
    return out


def bf_discounted(r, boot, term, trunc, tv, g):
    N, T = r.shape
    out = np.zeros((N, T))
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            h = K - t + 1
            out[n, t] = sum(g ** j * float(r[n, t + j]) for j in range(h)) + g ** h * nvK
    return out


def bf_td_lambda(r, v, boot, term, trunc, tv, g, lam):
    """Lambda-return as the (1-lam)-weighted average of n-step returns."""
    N, T = r.shape
    out = np.zeros((N, T))
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            h = K - t + 1

            def nstep(m):
                rew = sum(g ** j * float(r[n, t + j]) for j in range(m))
                tail = float(v[n, t + m]) if m < h else nvK
                return rew + g ** m * tail

            s = sum((1 - lam) * lam ** (m - 1) * nstep(m) for m in range(1, h))
            out[n, t] = s + lam ** (h - 1) * nstep(h)
    return out


def bf_vtrace(lr, r, v, boot, term, trunc, tv, g, lam, rho_bar, c_bar):
    N, T = r.shape
    vs = np.zeros((N, T))
    pg = np.zeros((N, T))
    ratio = np.exp(lr.astype(np.float64))
    rho = np.minimum(rho_bar, ratio)
    c = lam * np.minimum(c_bar, ratio)
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            s = 0.0
            for u in range(t, K + 1):
                succ = float(v[n, u + 1]) if u < K else nvK
                delta = rho[n, u] * (float(r[n, u]) + g * succ - float(v[n, u]))
                s += g ** (u - t) * np.prod(c[n, t:u]) * delta
            vs[n, t] = float(v[n, t]) + s
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            succ_vs = vs[n, t + 1] if t < K else nvK
            pg[n, t] = rho[n, t] * (float(r[n, t]) + g * succ_vs - float(v[n, t]))
    return vs, pg


def bf_retrace(q, pi, mu, act, r, boot, term, trunc, tv, g, lam):
    """Munos et al. off-policy sum: Qret_t = q_t + sum_s g^(s-t) (prod_{i=t+1..s} c_i) d_s."""
    N, T, A = q.shape
    q64, pi64 = q.astype(np.float64), pi.astype(np.float64)
    E = (q64 * pi64).sum(-1)
    qa = np.take_along_axis(q64, act[..., None].astype(np.int64), -1)[..., 0]
    pa = np.take_along_axis(pi64, act[..., None].astype(np.int64), -1)[..., 0]
    c = lam * np.minimum(1.0, pa / mu.astype(np.float64))
    out = np.zeros((N, T))
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, term[n], None if trunc is None else trunc[n])
            nvK = _nv(K, n, term[n], None if trunc is None else trunc[n],
                      None if tv is None else tv[n], boot)
            s = 0.0
            for u in range(t, K + 1):
                succ = E[n, u + 1] if u < K else nvK
                d = float(r[n, u]) + g * succ - qa[n, u]
                s += g ** (u - t) * np.prod(c[n, t + 1:u + 1]) * d
            out[n, t] = qa[n, t] + s
    return out


def _episode_start(t, term, trunc):
    j = t
    while j > 0 and not (term[j - 1] or (trunc is not None and trunc[j - 1])):
        j -= 1
    return j


def bf_elig(gin, init, term, trunc, g, lam):
    N, T = gin.shape
    out = np.zeros((N, T))
    for n in range(N):
        for t in range(T):
            st = _episode_start(t, term[n], None if trunc is None else trunc[n])
            s = sum((g * lam) ** (t - k) * float(gin[n, k]) for k in range(st, t + 1))
            if st == 0 and init is not None:
                s += (g * lam) ** (t + 1) * float(init[n])
            out[n, t] = s
    return out


def bf_prefix(x, term, trunc):
    N, T = x.shape
    out = np.zeros((N, T), np.int64)
    for n in range(N):
        for t in range(T):
            st = _episode_start(t, term[n], None if trunc is None else trunc[n])
            out[n, t] = int(x[n, st:t + 1].astype(np.int64).sum())
    return out


# --------------------------------------------------------------------------
# flag-pattern fixtures
# --------------------------------------------------------------------------

def _patterns():
    """Rows covering every termination pattern of length 8, every
    {none, term, trunc} pattern of length 8 restricted to 5 free steps, and
    random patterns with term and trunc on the same step."""
    rows_term, rows_trunc = [], []
    for bits in itertools.product([0, 1], repeat=8):
        rows_term.append(bits)
        rows_trunc.append((0,) * 8)
    for states in itertools.product([0, 1, 2], repeat=5):
        full = list(states) + [0, 0, 0]
        rows_term.append(tuple(1 if s == 1 else 0 for s in full))
        rows_trunc.append(tuple(1 if s == 2 else 0 for s in full))
    rng = np.random.default_rng(7)
    for _ in range(64):
        te = rng.random(8) < 0.3
        tr = rng.random(8) < 0.3
        rows_term.append(tuple(int(x) for x in te))
        rows_trunc.append(tuple(int(x) for x in tr))
    return np.array(rows_term, np.uint8), np.array(rows_trunc, np.uint8)


TERM, TRUNC = _patterns()
NP = TERM.shape[0]


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(rng, *shape):
    return rng.standard_normal(shape).astype(np.float32)


def _close(a, b, tol=1e-11):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    np.testing.assert_allclose(a, b, rtol=tol, atol=tol)


# --------------------------------------------------------------------------
# brute-force pins on exhaustive patterns
# --------------------------------------------------------------------------

def test_gae_matches_bruteforce_sum():
    rng = _rng(1)
    r, v, tv = _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP, 8)
    boot = _f32(rng, NP)
    adv, ret = oracle.gae(r, v, boot, TERM, TRUNC, tv, gamma=G, lam=L)
    ref = bf_gae(r, v, boot, TERM, TRUNC, tv, G, L)
    _close(adv, ref)
    _close(ret, ref + v.astype(np.float64))


def test_discounted_matches_bruteforce_sum():
    rng = _rng(2)
    r, tv, boot = _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP)
    _close(oracle.discounted_return(r, boot, TERM, TRUNC, tv, gamma=G),
           bf_discounted(r, boot, TERM, TRUNC, tv, G))
    # NULL bootstrap means a zero successor value at the window end
    _close(oracle.discounted_return(r, None, TERM, TRUNC, tv, gamma=G),
           bf_discounted(r, None, TERM, TRUNC, tv, G))


def test_td_lambda_matches_nstep_average():
    rng = _rng(3)
    r, v, tv, boot = _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP)
    _close(oracle.td_lambda(r, v, boot, TERM, TRUNC, tv, gamma=G, lam=L),
           bf_td_lambda(r, v, boot, TERM, TRUNC, tv, G, L))


@pytest.mark.parametrize("lam,rho_bar,c_bar", [(1.0, 1.0, 1.0), (0.95, 1.0, 0.9), (0.7, 2.0, 1.5)])
def test_vtrace_matches_impala_sum(lam, rho_bar, c_bar):
    rng = _rng(4)
    lr = (0.5 * _f32(rng, NP, 8)).astype(np.float32)
    r, v, tv, boot = _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP, 8), _f32(rng, NP)
    vs, pg = oracle.vtrace(lr, r, v, boot, TERM, TRUNC, tv, gamma=G, lam=lam,
                           rho_bar=rho_bar, c_bar=c_bar)
    vs_ref, pg_ref = bf_vtrace(lr, r, v, boot, TERM, TRUNC, tv, G, lam, rho_bar, c_bar)
    _close(vs, vs_ref)
    _close(pg, pg_ref)


@pytest.mark.parametrize("A", [1, 3, 6])
def test_retrace_matches_munos_sum(A):
    rng = _rng(5 + A)
    d = synthetic.make_inputs("retrace", NP, 8, seed=11 + A, A=A)
    tv = _f32(rng, NP, 8)
    out = oracle.retrace(d["q"], d["pi"], d["mu_a"], d["actions"], d["rewards"], d["bootstrap"],
                         TERM, TRUNC, tv, gamma=G, lam=L)
    ref = bf_retrace(d["q"], d["pi"], d["mu_a"], d["actions"], d["rewards"], d["bootstrap"],
                     TERM, TRUNC, tv, G, L)
    _close(out, ref)


@pytest.mark.parametrize("with_init", [False, True])
def test_elig_matches_episode_sum(with_init):
    rng = _rng(6)
    gin = _f32(rng, NP, 8)
    init = _f32(rng, NP) if with_init else None
    _close(oracle.elig_trace(gin, init, TERM, TRUNC, gamma=G, lam=L),
           bf_elig(gin, init, TERM, TRUNC, G, L))


def test_prefix_sum_matches_episode_sum():
    rng = _rng(7)
    x = rng.integers(-100, 101, size=(NP, 8)).astype(np.int32)
    out, mx = oracle.episodic_prefix_sum(x, TERM, TRUNC)
    ref = bf_prefix(x, TERM, TRUNC)
    np.testing.assert_array_equal(out.astype(np.int64), ref)
    assert mx == int(np.abs(ref).max())


def test_prefix_sum_wraps_twos_complement():
    # three steps of 2^30 overflow int32: the stored value is the low 32 bits
    x = np.full((1, 3), 1 << 30, np.int32)
    out, mx = oracle.episodic_prefix_sum(x, np.zeros((1, 3), np.uint8))
    assert mx == 3 << 30
    assert out[0, 2] == np.int64(3 << 30) - (1 << 32)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 5, 64])
def test_discounted_constant_reward_closed_form(T):
    g, r0, B = 0.97, 1.5, 0.25
    r = np.full((1, T), r0, np.float32)
    te = np.zeros((1, T), np.uint8)
    t = np.arange(T)
    out = oracle.discounted_return(r, None, te, gamma=g)
    _close(out[0], r0 * (1 - g ** (T - t)) / (1 - g), 1e-12)
    outb = oracle.discounted_return(r, np.array([B], np.float32), te, gamma=g)
    _close(outb[0], r0 * (1 - g ** (T - t)) / (1 - g) + g ** (T - t) * B, 1e-12)


def test_gae_constant_inputs_closed_form():
    T, g, lam, c0, V = 40, 0.99, 0.95, 0.5, 2.0
    te = np.zeros((1, T), np.uint8)
    t = np.arange(T)
    gl = g * lam
    # v = 0, boot = 0: delta = r, A_t = r (1 - (g lam)^(T-t)) / (1 - g lam)
    adv, _ = oracle.gae(np.full((1, T), c0, np.float32), np.zeros((1, T), np.float32),
                        np.zeros(1, np.float32), te, gamma=g, lam=lam)
    _close(adv[0], c0 * (1 - gl ** (T - t)) / (1 - gl), 1e-12)
    # r = 0, v = boot = V: delta = (g - 1) V
    adv, _ = oracle.gae(np.zeros((1, T), np.float32), np.full((1, T), V, np.float32),
                        np.full(1, V, np.float32), te, gamma=g, lam=lam)
    _close(adv[0], (g - 1) * V * (1 - gl ** (T - t)) / (1 - gl), 1e-12)


def test_elig_constant_input_closed_form():
    T, g, lam, g0, e0 = 50, 0.9, 0.9, 0.75, -1.25
    te = np.zeros((1, T), np.uint8)
    t = np.arange(T)
    gl = g * lam
    out = oracle.elig_trace(np.full((1, T), g0, np.float32), np.array([e0], np.float32), te,
                            gamma=g, lam=lam)
    _close(out[0], g0 * (1 - gl ** (t + 1)) / (1 - gl) + gl ** (t + 1) * e0, 1e-12)


def test_prefix_sum_counts_steps_since_reset():
    T = 30
    te = np.zeros((1, T), np.uint8)
    te[0, [4, 11, 12, 29]] = 1
    out, _ = oracle.episodic_prefix_sum(np.ones((1, T), np.int32), te)
    last_reset = 0
    for t in range(T):
        if t > 0 and te[0, t - 1]:
            last_reset = t
        assert out[0, t] == t - last_reset + 1


def test_gamma_zero_gives_local_terms():
    d = synthetic.make_inputs("vtrace", 16, 9, seed=3, p_term=0.2, p_trunc=0.2)
    r, v = d["rewards"].astype(np.float64), d["values"].astype(np.float64)
    rho = np.minimum(1.0, np.exp(d["log_rhos"].astype(np.float64)))
    args = (d["bootstrap"], d["terminated"], d["truncated"], d["trunc_value"])
    adv, _ = oracle.gae(d["rewards"], d["values"], *args, gamma=0.0, lam=0.9)
    _close(adv, r - v)
    _close(oracle.td_lambda(d["rewards"], d["values"], *args, gamma=0.0, lam=0.9), r)
    _close(oracle.discounted_return(d["rewards"], *args, gamma=0.0), r)
    vs, pg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], *args, gamma=0.0, lam=1.0)
    _close(vs - v, rho * (r - v))
    _close(pg, rho * (r - v))
    e = synthetic.make_inputs("retrace", 16, 9, seed=4, A=5, p_term=0.2)
    qr = oracle.retrace(e["q"], e["pi"], e["mu_a"], e["actions"], e["rewards"], e["bootstrap"],
                        e["terminated"], gamma=0.0, lam=0.9)
    _close(qr, e["rewards"])


# --------------------------------------------------------------------------
# cross-estimator identities
# --------------------------------------------------------------------------

def _sample(est, N=48, T=37, seed=21, **kw):
    kw.setdefault("p_term", 0.05)
    kw.setdefault("p_trunc", 0.05)
    return synthetic.make_inputs(est, N, T, seed=seed, **kw)


def test_gae_returns_equal_td_lambda_returns():
    d = _sample("gae")
    args = (d["rewards"], d["values"], d["bootstrap"], d["terminated"], d["truncated"],
            d["trunc_value"])
    for lam in (0.0, 0.5, 0.95, 1.0):
        _, ret = oracle.gae(*args, gamma=0.97, lam=lam)
        _close(ret, oracle.td_lambda(*args, gamma=0.97, lam=lam), 1e-10)


def test_gae_lambda_one_plus_value_is_discounted_return():
    d = _sample("gae", seed=22)
    adv, _ = oracle.gae(d["rewards"], d["values"], d["bootstrap"], d["terminated"],
                        d["truncated"], d["trunc_value"], gamma=0.97, lam=1.0)
    disc = oracle.discounted_return(d["rewards"], d["bootstrap"], d["terminated"],
                                    d["truncated"], d["trunc_value"], gamma=0.97)
    _close(adv + d["values"].astype(np.float64), disc, 1e-10)


@pytest.mark.parametrize("lam", [0.0, 0.6, 1.0])
def test_vtrace_on_policy_equals_td_lambda(lam):
    d = _sample("vtrace", seed=23)
    args = (d["rewards"], d["values"], d["bootstrap"], d["terminated"], d["truncated"],
            d["trunc_value"])
    vs, pg = oracle.vtrace(np.zeros_like(d["log_rhos"]), *args, gamma=0.97, lam=lam,
                           rho_bar=1.0, c_bar=1.0)
    _close(vs, oracle.td_lambda(*args, gamma=0.97, lam=lam), 1e-10)
    # with rho = 1 the pg advantage is the one-step target on vs minus V
    if lam == 1.0:
        _, ret = oracle.gae(*args, gamma=0.97, lam=1.0)
        _close(vs, ret, 1e-10)


def test_retrace_one_hot_policy_equals_td_lambda_on_q():
    N, T, A = 40, 33, 4
    d = _sample("retrace", N=N, T=T, seed=24, A=A)
    pi = np.zeros((N, T, A), np.float32)
    np.put_along_axis(pi, d["actions"][..., None].astype(np.int64), 1.0, -1)
    mu = np.ones((N, T), np.float32)
    for lam in (0.0, 0.7, 1.0):
        qr = oracle.retrace(d["q"], pi, mu, d["actions"], d["rewards"], d["bootstrap"],
                            d["terminated"], d["truncated"], d["trunc_value"], gamma=0.95, lam=lam)
        qa = np.take_along_axis(d["q"], d["actions"][..., None].astype(np.int64), -1)[..., 0]
        td = oracle.td_lambda(d["rewards"], qa, d["bootstrap"], d["terminated"], d["truncated"],
                              d["trunc_value"], gamma=0.95, lam=lam)
        _close(qr, td, 1e-10)


def test_retrace_lambda_zero_is_expected_sarsa():
    N, T, A = 20, 17, 5
    d = _sample("retrace", N=N, T=T, seed=25, A=A)
    qr = oracle.retrace(d["q"], d["pi"], d["mu_a"], d["actions"], d["rewards"], d["bootstrap"],
                        d["terminated"], d["truncated"], d["trunc_value"], gamma=0.9, lam=0.0)
    E = (d["q"].astype(np.float64) * d["pi"].astype(np.float64)).sum(-1)
    # expected-SARSA target: r_t + g E_{t+1}, boundary rules as for the value estimators
    td0 = oracle.td_lambda(d["rewards"], E.astype(np.float32), d["bootstrap"], d["terminated"],
                           d["truncated"], d["trunc_value"], gamma=0.9, lam=0.0)
    # td_lambda reads E as fp32; recompute the exact fp64 target directly
    ref = np.empty_like(td0)
    for n in range(N):
        for t in range(T):
            K = _boundary(t, T, d["terminated"][n], d["truncated"][n])
            succ = E[n, t + 1] if t < K else _nv(K, n, d["terminated"][n], d["truncated"][n],
                                                 d["trunc_value"][n], d["bootstrap"])
            ref[n, t] = float(d["rewards"][n, t]) + 0.9 * succ
    _close(qr, ref, 1e-10)
    np.testing.assert_allclose(qr, td0, rtol=1e-6, atol=1e-6)


def test_elig_unit_discount_on_integers_equals_prefix_sum():
    d = _sample("episodic_prefix_sum", seed=26)
    e = oracle.elig_trace(d["x"].astype(np.float32), None, d["terminated"], d["truncated"],
                          gamma=1.0, lam=1.0)
    s, _ = oracle.episodic_prefix_sum(d["x"], d["terminated"], d["truncated"])
    np.testing.assert_array_equal(e, s.astype(np.float64))


# --------------------------------------------------------------------------
# episode isolation: no signal crosses a done flag or a row
# --------------------------------------------------------------------------

@pytest.mark.parametrize("est", synthetic.ESTIMATORS)
def test_done_isolates_episodes(est):
    N, T, A = 6, 24, 3
    d = synthetic.make_inputs(est, N, T, seed=31, p_term=0.0, A=A)
    d["terminated"] = np.zeros((N, T), np.uint8)
    d["terminated"][:, 11] = 1        # boundary after step 11
    scal = synthetic.SCALARS[est]
    base = oracle.run(est, d, **scal)
    base = base if isinstance(base, tuple) else (base,)
    backward = est not in ("elig_trace", "episodic_prefix_sum")
    # perturb the side that must NOT influence the other: for backward
    # estimators the later episode (t >= 12) must not change t <= 11 ... except
    # through nothing at all, since step 11 terminates (successor value 0).
    other = slice(12, T) if backward else slice(0, 12)
    kept = slice(0, 12) if backward else slice(12, T)
    d2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in d.items()}
    for k in ("rewards", "values", "log_rhos", "inputs", "x", "q", "pi", "mu_a"):
        if k in d2 and d2[k] is not None:
            arr = d2[k]
            arr[:, other] = (arr[:, other] * 3 + 1).astype(arr.dtype)
    if "actions" in d2:
        d2["actions"][:, other] = (d2["actions"][:, other] + 1) % A
    # rows are independent too: perturb row 0 everywhere
    for k in ("rewards", "values", "inputs", "x", "q"):
        if k in d2 and d2[k] is not None:
            d2[k][0] = (d2[k][0] * 2 - 1).astype(d2[k].dtype)
    pert = oracle.run(est, d2, **scal)
    pert = pert if isinstance(pert, tuple) else (pert,)
    for a, b in zip(base, pert):
        if not isinstance(a, np.ndarray):
            continue
        np.testing.assert_array_equal(a[1:, kept], b[1:, kept])


def test_prefix_sum_stays_in_int32_at_workload_sizes():
    # |S| <= 100 * T; the longest workload row is T = 16384
    d = synthetic.workload_inputs("long_256x16384", "episodic_prefix_sum")
    _, mx = oracle.episodic_prefix_sum(d["x"], d["terminated"], d["truncated"])
    assert mx < 2 ** 31 - 1


# --------------------------------------------------------------------------
# the generic affine scan x_t = b_t + a_t x_prev (unified recurrence,
# gist.science technical summary, Methodologie 1, coefficients given)
# --------------------------------------------------------------------------

def bf_affine(a, b, reset, init, reverse):
    """Non-recursive: x at scan position p is the sum, over the positions q of
    p's segment (back to the nearest reset, or the row start), of b_q times
    the product of a over (q, p]; when the segment reaches the row start
    without a reset, init times the product of a over [0, p] is added."""
    N, T = a.shape
    out = np.zeros((N, T))
    for n in range(N):
        idx = list(range(T - 1, -1, -1)) if reverse else list(range(T))
        rs = [bool(reset is not None and reset[n, t]) for t in idx]
        for pos in range(T):
            start = pos
            while start > 0 and not rs[start]:
                start -= 1
            total = 0.0
            for q in range(start, pos + 1):
                total += float(b[n, idx[q]]) * float(np.prod([float(a[n, idx[u]]) for u in range(q + 1, pos + 1)]))
            if not rs[start] and init is not None:
                total += float(init[n]) * float(np.prod([float(a[n, idx[u]]) for u in range(0, pos + 1)]))
            out[n, idx[pos]] = total
    return out


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("with_init", [False, True])
def test_affine_matches_bruteforce_sum(reverse, with_init):
    d = synthetic.make_affine_inputs(4, 9, seed=31, p_reset=0.2, with_init=with_init, a_low=-1.2, a_high=1.2)
    got = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse)
    np.testing.assert_allclose(got, bf_affine(d["a"], d["b"], d["reset"], d["init"], reverse),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("reverse", [False, True])
def test_affine_every_reset_pattern(reverse):
    T = 5
    rng = np.random.default_rng(5)
    a = rng.uniform(-1, 1, (1, T)).astype(np.float32)
    b = rng.standard_normal((1, T)).astype(np.float32)
    init = rng.standard_normal(1).astype(np.float32)
    for bits in itertools.product([0, 1], repeat=T):
        reset = np.array([bits], np.uint8)
        got = oracle.affine_scan(a, b, reset, init, reverse=reverse)
        np.testing.assert_allclose(got, bf_affine(a, b, reset, init, reverse), rtol=1e-12, atol=1e-12)


def test_affine_unit_coefficient_is_cumulative_sum():
    d = synthetic.make_affine_inputs(3, 50, seed=32, p_reset=0.0, with_init=False)
    ones = np.ones_like(d["a"])
    np.testing.assert_allclose(oracle.affine_scan(ones, d["b"]), np.cumsum(d["b"].astype(np.float64), axis=1),
                               rtol=1e-12, atol=1e-12)
    rev = np.cumsum(d["b"][:, ::-1].astype(np.float64), axis=1)[:, ::-1]
    np.testing.assert_allclose(oracle.affine_scan(ones, d["b"], reverse=True), rev, rtol=1e-12, atol=1e-12)


def test_affine_zero_coefficient_returns_b():
    d = synthetic.make_affine_inputs(2, 17, seed=33, p_reset=0.1)
    for rev in (False, True):
        got = oracle.affine_scan(np.zeros_like(d["a"]), d["b"], d["reset"], d["init"], reverse=rev)
        np.testing.assert_array_equal(got, d["b"].astype(np.float64))


@pytest.mark.parametrize("c", [0.5, 0.99, -0.7])
def test_affine_constant_coefficient_geometric_sum(c):
    T = 40
    a = np.full((1, T), c, np.float32)
    b = np.ones((1, T), np.float32)
    cc = float(np.float32(c))
    k = np.arange(T, dtype=np.float64)
    want = (1.0 - cc ** (k + 1)) / (1.0 - cc)
    np.testing.assert_allclose(oracle.affine_scan(a, b)[0], want, rtol=1e-12)
    np.testing.assert_allclose(oracle.affine_scan(a, b, reverse=True)[0], want[::-1], rtol=1e-12)


def test_affine_backward_is_forward_on_reversed_rows():
    d = synthetic.make_affine_inputs(5, 64, seed=34, p_reset=0.05)
    fl = lambda x: None if x is None else np.ascontiguousarray(x[:, ::-1])  # noqa: E731
    back = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=True)
    fwd = oracle.affine_scan(fl(d["a"]), fl(d["b"]), fl(d["reset"]), d["init"])
    np.testing.assert_array_equal(back, fwd[:, ::-1])


def test_affine_reproduces_discounted_return():
    # discounted return = backward scan with a = gamma cont, b = r + gamma (1 - cont) nv
    d = synthetic.make_inputs("discounted_return", 6, 30, seed=35, p_term=0.1)
    r, term, boot = d["rewards"], d["terminated"], d["bootstrap"]
    g = float(np.float32(0.97))
    want = oracle.discounted_return(r, boot, term, None, None, gamma=g)
    cont = (term == 0).astype(np.float64)
    cont[:, -1] = 0.0
    nv = np.where(term != 0, 0.0, np.broadcast_to(boot.astype(np.float64)[:, None], r.shape))
    a = (g * cont).astype(np.float64)
    b = r.astype(np.float64) + g * (1.0 - cont) * nv
    got = bf_affine(a, b, None, None, reverse=True)
    np.testing.assert_allclose(want, got, rtol=1e-9, atol=1e-9)
    # and the oracle's own scan on the same (fp32-representable) coefficients
    a32, b32 = a.astype(np.float32), b.astype(np.float32)
    np.testing.assert_allclose(oracle.affine_scan(a32, b32, reverse=True), bf_affine(a32, b32, None, None, True),
                               rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# adjoint of the affine scan: pinned against central finite differences of
# the non-recursive forward sum (bf_affine), never against its own recursion
# --------------------------------------------------------------------------

def _fd_grads(a, b, reset, init, w, reverse, h=1e-5):
    """Gradients of L = sum(w * x) by central differences of bf_affine in fp64."""
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    i64 = None if init is None else init.astype(np.float64)
    L = lambda aa, bb, ii: float(np.sum(w * bf_affine(aa, bb, reset, ii, reverse)))  # noqa: E731
    da, db = np.zeros_like(a64), np.zeros_like(b64)
    for idx in np.ndindex(*a.shape):
        for arr, out in ((a64, da), (b64, db)):
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args_p = (p, b64, i64) if arr is a64 else (a64, p, i64)
            args_m = (m, b64, i64) if arr is a64 else (a64, m, i64)
            out[idx] = (L(*args_p) - L(*args_m)) / (2 * h)
    dinit = np.zeros(a.shape[0])
    if i64 is not None:
        for n in range(a.shape[0]):
            p, m = i64.copy(), i64.copy()
            p[n] += h
            m[n] -= h
            dinit[n] = (L(a64, b64, p) - L(a64, b64, m)) / (2 * h)
    return da, db, dinit


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("p_reset", [0.0, 0.3])
def test_affine_grad_matches_finite_differences(reverse, p_reset):
    d = synthetic.make_affine_inputs(3, 7, seed=41, p_reset=p_reset, a_low=-1.1, a_high=1.1)
    w = np.random.default_rng(42).standard_normal((3, 7)).astype(np.float32)
    x = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse).astype(np.float32)
    da, db, dinit = oracle.affine_scan_grad(d["a"], x, w, d["reset"], d["init"], reverse=reverse)
    fda, fdb, fdinit = _fd_grads(d["a"], d["b"], d["reset"], d["init"], w.astype(np.float64), reverse)
    np.testing.assert_allclose(db, fdb, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(da, fda, rtol=1e-5, atol=1e-5)  # x passed as fp32
    np.testing.assert_allclose(dinit, fdinit, rtol=1e-6, atol=1e-6)


def test_affine_grad_unit_coefficient_is_reverse_cumsum():
    d = synthetic.make_affine_inputs(2, 40, seed=43, p_reset=0.0, with_init=False)
    a = np.ones_like(d["a"])
    dy = d["b"]
    x = oracle.affine_scan(a, d["b"]).astype(np.float32)
    _, db, _ = oracle.affine_scan_grad(a, x, dy)
    np.testing.assert_allclose(db, np.cumsum(dy[:, ::-1].astype(np.float64), axis=1)[:, ::-1], rtol=1e-12)
    _, db_r, _ = oracle.affine_scan_grad(a, x, dy, reverse=True)
    np.testing.assert_allclose(db_r, np.cumsum(dy.astype(np.float64), axis=1), rtol=1e-12)


def test_affine_grad_zero_coefficient():
    d = synthetic.make_affine_inputs(2, 9, seed=44, p_reset=0.0)
    a = np.zeros_like(d["a"])
    x = oracle.affine_scan(a, d["b"], None, d["init"]).astype(np.float32)
    dy = d["b"]
    da, db, dinit = oracle.affine_scan_grad(a, x, dy, None, d["init"])
    np.testing.assert_array_equal(db, dy.astype(np.float64))
    xp = np.concatenate([d["init"][:, None], x[:, :-1]], axis=1).astype(np.float64)
    np.testing.assert_allclose(da, dy.astype(np.float64) * xp, rtol=1e-15)
    np.testing.assert_array_equal(dinit, np.zeros(2))


# --------------------------------------------------------------------------
# time-major affine scan ([T, N] arrays): pinned against the non-recursive
# sum on the transposed rows, and against the row-major routine
# --------------------------------------------------------------------------

@pytest.mark.parametrize("reverse", [False, True])
def test_affine_tm_matches_bruteforce_on_transpose(reverse):
    d = synthetic.make_affine_inputs(5, 9, seed=51, p_reset=0.2, a_low=-1.1, a_high=1.1)
    tm = lambda v: None if v is None else np.ascontiguousarray(v.T)  # noqa: E731
    got = oracle.affine_scan_tm(tm(d["a"]), tm(d["b"]), tm(d["reset"]), d["init"], reverse=reverse)
    want = bf_affine(d["a"], d["b"], d["reset"], d["init"], reverse)
    np.testing.assert_allclose(got, want.T, rtol=1e-12, atol=1e-12)


def test_affine_tm_is_row_major_on_transposed_arrays():
    d = synthetic.make_affine_inputs(7, 300, seed=52, p_reset=0.05)
    tm = lambda v: None if v is None else np.ascontiguousarray(v.T)  # noqa: E731
    for reverse in (False, True):
        got = oracle.affine_scan_tm(tm(d["a"]), tm(d["b"]), tm(d["reset"]), d["init"], reverse=reverse)
        want = oracle.affine_scan(d["a"], d["b"], d["reset"], d["init"], reverse=reverse)
        np.testing.assert_array_equal(got, want.T)
