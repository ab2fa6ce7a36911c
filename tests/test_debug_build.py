"""The bounds-checking build (liblighthouse_debug.so, -DLH_DEBUG=1).

The compute sanitizer is not available on this GPU pool, so the library has a
build of its own in which every kernel checks the indices it computes from data
(idx, pos, slot) or from unit, tile and level coordinates before the access,
and reports a failed check through lh_read_device_status (LH_STATUS_BOUNDS)
instead of trapping.

CPU: the debug library loads and exports every declared entry point; the
check predicates themselves (compiled for the host in liblh_selftest.so) accept
exactly the in-range indices -- out-of-range values are tried here, on the
CPU, and never given to a kernel.
GPU: the stage and fused parity tests of the small cases run again in a child
process against the debug library, with valid inputs only; after each of them
the device status must show no bounds failure (tests/conftest.py).
"""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from long_context_lh_b200 import build  # noqa: E402


def test_debug_library_exports_every_declared_symbol():
    from test_host import declared_functions
    lib = ctypes.CDLL(build.LIB_DEBUG)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} missing from the debug build"


def predicates():
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    f = lib.lh_selftest_bounds
    f.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
    f.restype = ctypes.c_int
    return lambda which, a, b, c=0: f(which, a, b, c)


def test_bounds_predicates_on_the_host():
    p = predicates()
    big = 1 << 40
    # in_range(v, n): 0 <= v < n
    for v, n, ok in ((0, 1, 1), (5, 6, 1), (6, 6, 0), (-1, 6, 0), (0, 0, 0), (big, big + 1, 1),
                     (big, big, 0), (-big, 3, 0)):
        assert p(0, v, n) == ok, (v, n)
    # slot_ok(s, S): -1 <= s < S
    for s_, S, ok in ((-1, 8, 1), (0, 8, 1), (7, 8, 1), (8, 8, 0), (-2, 8, 0), (-1, 1, 1),
                      (2 ** 31 - 1, 2 ** 31, 1), (-(2 ** 31), 8, 0)):
        assert p(1, s_, S) == ok, (s_, S)
    # rows_ok(first, count, n): [first, first + count) inside [0, n), no overflow
    for f, c, n, ok in ((0, 8, 8, 1), (1, 8, 8, 0), (8, 0, 8, 1), (9, 0, 8, 0), (-1, 1, 8, 0),
                        (0, -1, 8, 0), (2, 2 ** 62, 8, 0), (2 ** 62, 2 ** 62, 2 ** 62, 0)):
        assert p(2, f, c, n) == ok, (f, c, n)
    # entry_ok(j, off_l, off_next): off_l <= off_l + j < off_next
    for j, a, b, ok in ((0, 100, 101, 1), (1, 100, 101, 0), (-1, 100, 200, 0), (99, 100, 200, 1),
                        (100, 100, 200, 0)):
        assert p(3, j, a, b) == ok, (j, a, b)
    assert p(9, 0, 0) == -1


@pytest.mark.gpu
def test_stage_and_fused_calls_report_no_bounds_failure():
    env = dict(os.environ, LH_LIBRARY="debug", PYTHONPATH=ROOT)
    sel = ("front_stages or gather_and_scatter or pooled or attention_matches or fused_forward "
           "or variant or scatter_modes or degenerate or ties or deterministic or non_finite")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_parity_gpu.py"),
                        "-m", "gpu", "-x", "-k", sel, "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "liblighthouse_debug.so" in r.stdout, tail
