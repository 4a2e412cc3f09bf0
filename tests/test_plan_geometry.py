"""Host checks of the launch geometry (no GPU): the plans the library reports
(rlscan_query_plan / rlscan_query_plan_tm) against the index arithmetic the
kernels use, restated here.  Every access must stay inside its buffer, and the
ticket order must be a dependency order: a chunk only ever waits for chunks
whose tickets were drawn earlier (so a waiting block's predecessors are
already running, and no launch can deadlock)."""
import itertools

import pytest

import segmented_linear_recurrence_b200 as slr

K_TM = 8  # steps per thread of every time-major kernel


def tm_geometry(N, T):
    """(wt_log2, nct, nbc, dpitch) from the reported plan, as the kernel sees them."""
    p = slr.rlscan_query_plan_tm("gae", N, T)
    cols_times_span = p["chunk_steps"]  # (K << wl) * (256 >> wl) = 2048 for every wl
    assert cols_times_span == K_TM * 256
    wl = 0
    while wl < 3 and (K_TM << wl) < T:
        wl += 1
    span, cols = K_TM << wl, 256 >> wl
    nct, nbc = -(-T // span), -(-N // cols)
    assert p["chunks"] == nct * nbc
    assert p["lookback"] == (1 if nct > 1 else 0)
    dpitch = nbc * cols
    if nct > 1:
        assert p["workspace_bytes"] == 16 + 16 * nct * dpitch
    return wl, nct, nbc, dpitch


@pytest.mark.parametrize("N,T", [(1, 1), (5, 7), (33, 9), (96, 16), (300, 32), (257, 129), (4096, 512),
                                 (64, 2048), (2, 40001), (1000, 64), (130, 65)])
def test_time_major_accesses_stay_in_bounds(N, T):
    wl, nct, nbc, dpitch = tm_geometry(N, T)
    wt = 1 << wl
    for chunk in range(nct * nbc):
        for backward in (False, True):
            jd, cb = divmod(chunk, nbc)
            j = nct - 1 - jd if backward else jd
            for warp in range(8):
                slice_, group = warp & (wt - 1), warp >> wl
                for lane in (0, 31):
                    n = cb * (256 >> wl) + (group << 5) + lane
                    t0 = ((j << wl) + slice_) * K_TM
                    if n >= N or t0 >= T:
                        continue  # no access at all
                    last = min(T, t0 + K_TM) - 1
                    assert last * N + n < N * T  # every step load / store
                    if t0 + K_TM < T:  # halo (backward): step t0 + K
                        assert (t0 + K_TM) * N + n < N * T
                    if t0 > 0:  # halo (forward): step t0 - 1
                        assert (t0 - 1) * N + n >= 0
                    if nct > 1:
                        assert j * dpitch + n < nct * dpitch  # descriptor
    # each (environment, step) is owned by exactly one thread of one chunk
    owned = set()
    for chunk in range(nct * nbc):
        jd, cb = divmod(chunk, nbc)
        for warp in range(8):
            slice_, group = warp & (wt - 1), warp >> wl
            for lane in range(32):
                n = cb * (256 >> wl) + (group << 5) + lane
                t0 = ((jd << wl) + slice_) * K_TM
                for k in range(K_TM):
                    if n < N and t0 + k < T:
                        assert (n, t0 + k) not in owned
                        owned.add((n, t0 + k))
    assert len(owned) == N * T


def time_major_order_ok(N, T):
    wl, nct, nbc, _ = tm_geometry(N, T)
    for backward in (False, True):
        ticket_of = {}
        for t in range(nct * nbc):
            jd, cb = divmod(t, nbc)
            ticket_of[(nct - 1 - jd if backward else jd, cb)] = t
        for (j, cb), t in ticket_of.items():
            pred = j + 1 if backward else j - 1
            if 0 <= pred < nct:
                assert ticket_of[(pred, cb)] < t
    return True


@pytest.mark.parametrize("N,T", [(96, 1000), (5, 700), (300, 129)])
def test_time_major_tickets_are_a_dependency_order(N, T):
    assert time_major_order_ok(N, T)


def chunk_of_ticket(nchunks, cpr, ticket, backward):
    """Row-major look-back plan: the chunk a ticket stands for (scan_kernel.cuh)."""
    if cpr == 0:
        return nchunks - 1 - ticket if backward else ticket
    rows = nchunks // cpr
    s, r = divmod(ticket, rows)
    return r * cpr + (cpr - 1 - s if backward else s)


@pytest.mark.parametrize("est,N,T", [("gae", 37, 16384), ("gae", 3, 6144), ("elig_trace", 130, 12288),
                                     ("elig_trace", 3, 10000), ("retrace", 9, 8192), ("vtrace", 5, 5000)])
def test_row_major_tickets_are_a_dependency_order(est, N, T):
    p = slr.rlscan_query_plan(est, N, T, 6)
    assert p["lookback"] == 1 and p["launches"] == 1
    L, nchunks = p["chunk_steps"], p["chunks"]
    cpr = T // L if T % L == 0 else 0
    assert nchunks == -(-N * T // L)
    for backward in (False, True):
        chunks = [chunk_of_ticket(nchunks, cpr, t, backward) for t in range(nchunks)]
        assert sorted(chunks) == list(range(nchunks))  # a bijection
        ticket = {c: t for t, c in enumerate(chunks)}
        for c in range(nchunks):
            pred = c + 1 if backward else c - 1  # the chunk whose carry c needs
            if not 0 <= pred < nchunks:
                continue
            # a chunk whose dependency edge is a row boundary needs no carry
            edge = (min((c + 1) * L, N * T) % T == 0) if backward else ((c * L) % T == 0)
            if not edge:
                assert ticket[pred] < ticket[c], (c, pred)
