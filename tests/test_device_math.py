"""The FMA-pipe exponential of the forward attention (ex2_fma2, tc_common.cuh).

CPU: the committed Remez fit (csrc/fit_ex2_poly.py) reproduces the kernel's four
fp32 constants, and its fp32 Horner evaluation stays within the stated
7.5e-5 relative error of 2^f on [-1/2, 1/2].
GPU: the device function itself (through liblh_selftest.so, a test-only
library) against exp2 in fp64 over [-125, 8], with the integers and the
half-integers where the reduction changes n, and the clamp below -125.
"""
import ctypes
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_context_lh_b200", "csrc")
BOUND = 7.5e-5  # stated in tc_common.cuh


def fit_module():
    spec = importlib.util.spec_from_file_location("fit_ex2_poly", os.path.join(CSRC, "fit_ex2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def kernel_constants():
    src = open(os.path.join(CSRC, "tc_common.cuh")).read()
    body = src[src.index("ex2_fma2(float2 x)"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f,", body)]
    # Horner order in the kernel: c3 (with c2), then c1, then c0
    c3, c2, c1, c0 = vals[-4:]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_fit_reproduces_the_kernel_constants():
    m = fit_module()
    got = m.fitted_constants()
    assert np.array_equal(got, kernel_constants()), (got, kernel_constants())
    assert m.fp32_poly_max_rel_error(got) <= BOUND


def test_fit_is_a_minimax_fit():
    """Equioscillation (what makes it the minimax polynomial): the relative error
    reaches its maximum magnitude with alternating signs at deg + 2 = 5 points."""
    m = fit_module()
    c = m.remez_relative()
    g = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
    E = np.abs(e).max()
    peaks = g[np.abs(e) > E * (1 - 1e-6)]
    # cluster the near-maximal points and read the sign at each cluster
    signs = []
    last = None
    for x in peaks:
        if last is None or x - last > 1e-3:
            signs.append(np.sign(np.polyval(c[::-1], x) / np.exp2(x) - 1.0))
        last = x
    assert len(signs) == 5 and all(signs[i] == -signs[i + 1] for i in range(4)), signs


@pytest.mark.gpu
def test_device_ex2_fma2_within_its_bound():
    import torch
    from long_context_lh_b200 import build
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    lib.lh_selftest_ex2_fma2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    lib.lh_selftest_ex2_fma2.restype = ctypes.c_int
    ints = np.arange(-125, 9, dtype=np.float64)
    halves = ints[:-1] + 0.5
    near = np.concatenate([np.nextafter(halves.astype(np.float32), np.float32(-1e9)),
                           np.nextafter(halves.astype(np.float32), np.float32(1e9))])
    x = np.concatenate([np.linspace(-125.0, 8.0, 1 << 22), ints, halves, near,
                        np.linspace(-200.0, -125.0, 1001)]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    dev = torch.device("cuda:0")
    xd = torch.from_numpy(x).to(dev)
    yd = torch.empty_like(xd)
    assert lib.lh_selftest_ex2_fma2(xd.data_ptr(), yd.data_ptr(), xd.numel(), None) == 0
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    x64 = x.astype(np.float64)
    inr = x64 >= -125.0
    rel = np.abs(y[inr] / np.exp2(x64[inr]) - 1.0)
    assert rel.max() <= BOUND, f"max relative error {rel.max():.4g} at x={x64[inr][np.argmax(rel)]}"
    # below -125 the argument is clamped: every value equals the value at -125
    y125 = y[np.where(x64 == -125.0)[0][0]]
    assert np.all(y[~inr] == y125)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
