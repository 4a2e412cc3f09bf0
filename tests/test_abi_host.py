"""Host-only checks of the C ABI boundary (no GPU needed).

The library must load, export every entry point include/rlscan.h declares,
and reject invalid arguments synchronously -- before any CUDA call -- with the
documented status codes.  Fake (never dereferenced) addresses are used for
the pointers: argument checks run before anything touches them.
"""
import ctypes
import os
import re

import pytest

import segmented_linear_recurrence_b200 as slr
from segmented_linear_recurrence_b200 import build as slr_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rlscan.h")

OK, INVALID, OVERLAP = 0, 1, 2


@pytest.fixture(scope="module")
def L():
    slr_build.build()
    return slr.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rlscan_\w+)\s*\(", src)))


def test_header_declares_the_seven_estimators():
    names = declared_functions()
    for est in ("gae", "vtrace", "retrace", "td_lambda", "discounted_return", "elig_trace",
                "episodic_prefix_sum"):
        assert f"rlscan_{est}" in names


def test_library_exports_every_declared_symbol(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", slr.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (rlscan_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(L, n)


def test_abi_version_and_status_strings(L):
    assert slr.rlscan_abi_version() == 1
    for code, name in slr.STATUS.items():
        assert slr.rlscan_status_string(code) == name
    assert slr.rlscan_status_string(99) == "RLSCAN_ERR_UNKNOWN"


def P(addr):
    return ctypes.c_void_p(addr)


BASE = 0x7F0000000000  # a fake, 256-byte aligned address range; never dereferenced


def gae(L, N=4, T=8, r=BASE, v=BASE + 0x10000, b=BASE + 0x20000, te=BASE + 0x30000, tr=None,
        tv=None, adv=BASE + 0x40000, ret=BASE + 0x50000, g=0.99, lam=0.95):
    return L.rlscan_gae(P(r), P(v), P(b), P(te) if te else None, P(tr) if tr else None,
                        P(tv) if tv else None, P(adv) if adv else None, P(ret) if ret else None,
                        N, T, g, lam, None)


def test_empty_problem_is_a_noop(L):
    assert gae(L, N=0, T=8, r=0, v=0, b=0, te=0, adv=0, ret=0) == OK
    assert gae(L, N=5, T=0, r=0, v=0, b=0, te=0, adv=0, ret=0) == OK
    assert L.rlscan_episodic_prefix_sum(None, None, None, None, 0, 0, None) == OK


def test_negative_sizes_rejected(L):
    assert gae(L, N=-1) == INVALID
    assert gae(L, T=-3) == INVALID


def test_null_mandatory_pointers_rejected(L):
    assert gae(L, r=0) == INVALID
    assert gae(L, v=0) == INVALID
    assert gae(L, b=0) == INVALID
    assert gae(L, adv=0) == INVALID
    # truncated given without trunc_value
    assert gae(L, tr=BASE + 0x60000, tv=0) == INVALID


def test_misaligned_float_pointer_rejected(L):
    assert gae(L, r=BASE + 2) == INVALID


def test_non_finite_scalars_rejected(L):
    assert gae(L, g=float("nan")) == INVALID
    assert gae(L, lam=float("inf")) == INVALID
    vp = [P(BASE + i * 0x10000) for i in range(9)]
    st = L.rlscan_vtrace(vp[0], vp[1], vp[2], vp[3], vp[4], None, None, vp[5], vp[6], 4, 8, 0.99,
                         1.0, 0.0, 1.0, None)
    assert st == INVALID  # rho_bar must be > 0


def test_overlapping_outputs_rejected(L):
    # output overlapping an input (in-place) and two overlapping outputs
    assert gae(L, adv=BASE) == OVERLAP
    assert gae(L, ret=BASE + 0x40000 + 16) == OVERLAP
    # adjacent, non-overlapping buffers are fine up to the device check
    N, T = 4, 8
    st = gae(L, N=N, T=T, adv=BASE + 0x40000, ret=BASE + 0x40000 + N * T * 4)
    assert st != OVERLAP


def test_retrace_action_dim_limits(L):
    vp = [P(BASE + i * 0x100000) for i in range(10)]
    args = vp[:9] + [vp[9]]
    assert L.rlscan_retrace(*args, 4, 8, 0, 0.99, 0.95, None) == INVALID
    assert L.rlscan_retrace(*args, 4, 8, 4096, 0.99, 0.95, None) == INVALID
    assert L.rlscan_retrace(*args, 2, 1 << 20, 1 << 11, 0.99, 0.95, None) == INVALID  # T*A > 2^30


def test_valid_call_without_gpu_reports_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert gae(L) not in (OK, INVALID, OVERLAP)


def test_query_plan(L):
    p = slr.rlscan_query_plan("gae", 4096, 512)
    assert p["lookback"] == 0 and p["chunk_steps"] % 512 == 0 and p["launches"] == 1
    assert p["chunks"] == 4096 * 512 // p["chunk_steps"]
    p = slr.rlscan_query_plan("vtrace", 256, 16384)
    assert p["lookback"] == 1 and p["workspace_bytes"] >= 16 * p["chunks"]
    p = slr.rlscan_query_plan("retrace", 2048, 512, 18)
    assert p["lookback"] == 0 and p["block_threads"] in (128, 256)
    # rows that do not divide a block still get whole-row blocks
    p = slr.rlscan_query_plan("episodic_prefix_sum", 3, 33)
    assert p["lookback"] == 0 and p["chunk_steps"] % 33 == 0 and p["chunks"] == 1
    p = slr.rlscan_query_plan("gae", 4096, 2000)
    assert p["lookback"] == 0 and p["chunk_steps"] % 2000 == 0
    assert p["chunks"] == -(-4096 // (p["chunk_steps"] // 2000))
    # the block size whose threads whole rows fill best
    assert slr.rlscan_query_plan("gae", 64, 3000)["block_threads"] == 384
    assert slr.rlscan_query_plan("gae", 64, 1500)["block_threads"] == 192
    # a row longer than the largest block needs the look-back
    assert slr.rlscan_query_plan("gae", 8, 4097)["lookback"] == 1
    assert slr.rlscan_query_plan("gae", 8, 4096)["lookback"] == 0
    # more steps than one launch takes are split by rows
    p = slr.rlscan_query_plan("discounted_return", 1 << 12, 1 << 19)
    assert p["launches"] == 2
    assert slr.rlscan_query_plan("gae", 0, 5)["chunks"] == 0


def test_options_roundtrip(L):
    for name, default in (("lookback_timeout_ns", 10 ** 9), ("force_lookback", 0),
                          ("force_block", 0), ("force_scalar", 0), ("check_pointers", 1),
                          ("test_starve_lookback", 0), ("pdl", 1)):
        assert slr.rlscan_get_option(name) == default
    slr.rlscan_set_option("force_block", 512)
    assert slr.rlscan_query_plan("gae", 64, 32)["block_threads"] == 512
    slr.rlscan_set_option("force_block", 0)
    slr.rlscan_set_option("force_block", 192)
    assert slr.rlscan_query_plan("gae", 64, 32)["block_threads"] == 192
    slr.rlscan_set_option("force_block", 0)
    for bad in (100, 200, 576, 1024):
        with pytest.raises(slr.RlscanError):
            slr.rlscan_set_option("force_block", bad)
    with pytest.raises(slr.RlscanError):
        slr.rlscan_set_option("lookback_timeout_ns", 10)
    slr.rlscan_set_option("force_lookback", 1)
    assert slr.rlscan_query_plan("gae", 64, 32)["lookback"] == 1
    slr.rlscan_set_option("force_lookback", 0)


def test_binding_raises_without_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    r = torch.zeros(2, 4)
    with pytest.raises(RuntimeError):
        slr.rlscan_discounted_return(r, None, torch.zeros(2, 4, dtype=torch.uint8))


def test_affine_scan_argument_checks(L):
    a, b, x = P(BASE), P(BASE + 0x10000), P(BASE + 0x20000)
    assert L.rlscan_affine_scan(None, None, None, None, None, 0, 5, 0, None) == OK  # empty
    assert L.rlscan_affine_scan(a, b, None, None, x, 4, 8, 2, None) == INVALID  # direction
    assert L.rlscan_affine_scan(a, b, None, None, x, 4, 8, -1, None) == INVALID
    assert L.rlscan_affine_scan(None, b, None, None, x, 4, 8, 0, None) == INVALID  # a required
    assert L.rlscan_affine_scan(a, None, None, None, x, 4, 8, 0, None) == INVALID  # b required
    assert L.rlscan_affine_scan(a, b, None, None, None, 4, 8, 1, None) == INVALID  # x required
    assert L.rlscan_affine_scan(a, b, None, None, P(BASE + 2), 4, 8, 1, None) == INVALID  # misaligned
    assert L.rlscan_affine_scan(a, b, None, None, a, 4, 8, 1, None) == OVERLAP  # in place
    p = slr.rlscan_query_plan("affine_scan", 4096, 2000)
    assert p["lookback"] == 0 and p["chunk_steps"] % 2000 == 0
    assert slr.rlscan_query_plan("affine_scan", 2, 100000)["lookback"] == 1


def test_affine_scan_bf16_argument_checks(L):
    a, b, x = P(BASE), P(BASE + 0x10000), P(BASE + 0x20000)
    assert L.rlscan_affine_scan_bf16(a, b, None, None, x, 4, 8, 3, None) == INVALID  # direction
    assert L.rlscan_affine_scan_bf16(a, b, None, None, P(BASE + 0x20001), 4, 8, 0, None) == INVALID  # odd address
    assert L.rlscan_affine_scan_bf16(a, b, None, None, b, 4, 8, 0, None) == OVERLAP
    assert slr.rlscan_query_plan("affine_scan_bf16", 4096, 2048)["lookback"] == 0


def test_time_major_argument_checks(L):
    r, v, b, o = P(BASE), P(BASE + 0x10000), P(BASE + 0x20000), P(BASE + 0x30000)
    te = P(BASE + 0x40000)
    assert L.rlscan_gae_tm(None, None, None, None, None, None, None, None, 0, 5, 0.99, 0.95, None) == OK
    assert L.rlscan_gae_tm(r, v, b, te, None, None, o, None, -1, 5, 0.99, 0.95, None) == INVALID
    assert L.rlscan_gae_tm(r, None, b, te, None, None, o, None, 4, 5, 0.99, 0.95, None) == INVALID
    assert L.rlscan_gae_tm(r, v, b, te, te, None, o, None, 4, 5, 0.99, 0.95, None) == INVALID  # trunc_value
    assert L.rlscan_gae_tm(r, v, b, te, None, None, r, None, 4, 5, 0.99, 0.95, None) == OVERLAP
    assert L.rlscan_gae_tm(r, v, b, te, None, None, P(BASE + 0x30002), None, 4, 5, 0.99, 0.95,
                           None) == INVALID  # misaligned
    assert L.rlscan_gae_tm(r, v, b, te, None, None, o, None, (1 << 26) + 1, 2, 0.99, 0.95,
                           None) == INVALID  # more environments than the layout takes
    assert L.rlscan_vtrace_tm(r, v, b, o, te, None, None, P(BASE + 0x50000), None, 4, 5, 0.99, 1.0, 0.0, 1.0,
                              None) == INVALID  # rho_bar
    assert L.rlscan_td_lambda_tm(r, v, b, te, None, None, o, 4, 5, float("nan"), 0.95, None) == INVALID
    assert L.rlscan_discounted_return_tm(None, None, te, None, None, o, 4, 5, 0.99, None) == INVALID
    assert L.rlscan_elig_trace_tm(r, None, te, None, r, 4, 5, 0.99, 0.95, None) == OVERLAP
    assert L.rlscan_episodic_prefix_sum_tm(r, te, None, None, 4, 5, None) == INVALID
    assert L.rlscan_affine_scan_tm(r, v, None, None, o, 4, 8, 2, None) == INVALID  # direction


def test_query_plan_time_major(L):
    # T <= 64: one chunk per column block of 256 / slices environments
    for T, cols in [(1, 256), (8, 256), (9, 128), (16, 128), (17, 64), (32, 64), (33, 32), (64, 32)]:
        p = slr.rlscan_query_plan_tm("gae", 1000, T)
        assert p["lookback"] == 0 and p["block_threads"] == 256 and p["launches"] == 1
        assert p["chunks"] == -(-1000 // cols), (T, p)
    # longer windows chain 64-step chunks of 32 environments
    p = slr.rlscan_query_plan_tm("vtrace", 4096, 2048)
    assert p["lookback"] == 1 and p["chunk_steps"] == 64 * 32 and p["chunks"] == 32 * 128
    assert p["workspace_bytes"] == 16 + 16 * 32 * 4096
    assert slr.rlscan_query_plan_tm("elig_trace", 33, 65)["chunks"] == 2 * 2
    # forced look-back halves the chunk while it stays below T
    slr.rlscan_set_option("force_lookback", 1)
    try:
        p = slr.rlscan_query_plan_tm("gae", 100, 32)
        assert p["lookback"] == 1 and p["chunks"] == 2  # 16-step chunks of 128 environments
    finally:
        slr.rlscan_set_option("force_lookback", 0)
    with pytest.raises(slr.RlscanError):
        slr.rlscan_query_plan_tm("retrace", 8, 8)
    assert slr.rlscan_query_plan_tm("affine_scan", 0, 5)["chunks"] == 0


def test_gae_bf16_argument_checks(L):
    r, v, b, o = P(BASE), P(BASE + 0x10000), P(BASE + 0x20000), P(BASE + 0x30000)
    assert L.rlscan_gae_bf16(None, None, None, None, None, None, None, None, 0, 5, 0.99, 0.95, None) == OK
    assert L.rlscan_gae_bf16(r, v, None, None, None, None, o, None, 4, 8, 0.99, 0.95, None) == INVALID  # bootstrap
    assert L.rlscan_gae_bf16(r, v, b, None, None, None, P(BASE + 0x30001), None, 4, 8, 0.99, 0.95,
                             None) == INVALID  # odd address
    assert L.rlscan_gae_bf16(r, v, b, None, None, None, v, None, 4, 8, 0.99, 0.95, None) == OVERLAP
    assert L.rlscan_gae_bf16(r, v, b, None, None, None, o, None, 4, 8, float("inf"), 0.95, None) == INVALID


def test_plain_c_program_uses_the_abi(tmp_path):
    # The header is C99 and the library links from C: a C user exercises the
    # device-free calls (version, strings, plans, options, argument checks).
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c", "abi_smoke.c")
    exe = tmp_path / "abi_smoke"
    libdir = os.path.dirname(slr.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    "-L", libdir, "-l:librlscan.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert "abi_smoke ok" in out.stdout


def test_layout_dispatch_decision():
    # The binding sends [N, T] views of time-major storage to the "_tm" path
    # and everything else to the row-major path (decided on the host).
    import torch
    from segmented_linear_recurrence_b200 import api
    seen = []

    def fake(*args, _tm=False, **kw):
        seen.append((_tm, [tuple(a.shape) for a in args if isinstance(a, torch.Tensor)]))
        first = next(a for a in args if isinstance(a, torch.Tensor) and a.dim() == 2)
        return first.clone(), None

    f = api._layout_dispatch(fake)
    buf_tm = torch.zeros(7, 5)          # [T, N] storage
    per_env = torch.zeros(5)
    out, none = f(buf_tm.T, buf_tm.T, per_env)
    assert seen[-1] == (True, [(7, 5), (7, 5), (5,)]) and none is None
    assert out.shape == (5, 7) and out.t().is_contiguous()   # [N, T] view of a [T, N] result
    f(torch.zeros(5, 7), torch.zeros(5, 7), per_env)         # row-major: untouched
    assert seen[-1] == (False, [(5, 7), (5, 7), (5,)])
    f(buf_tm.T, torch.zeros(5, 7), per_env)                  # mixed layouts: row-major path (which then rejects)
    assert seen[-1][0] is False
