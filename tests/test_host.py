"""Host-side checks of the C-ABI library (no GPU needed).

The library must load on a machine without a GPU, export every entry point the
header declares, and reject bad shapes/arguments on the host before any launch.
"""
import ctypes
import os
import re

import pytest

from long_context_lh_b200 import lighthouse as lh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lighthouse.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lh_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = lh._lib()
    names = declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), f"{n} declared in lighthouse.h but not exported"
    assert sorted(lh.EXPORTED) == names


def S(B=1, H=2, N=4096, d=64, p=4, L=3, S_=512):
    return lh.make_shape(B, H, N, d, p, L, S_)


def test_validate_accepts_the_workloads():
    for shp in (S(), S(1, 16, 98304, 64, 4, 4, 8192), S(1, 16, 524288, 64, 4, 5, 16384),
                S(1, 8, 1048576, 128, 4, 6, 16384), S(1, 1, 100, 64, 2, 1, 100)):
        assert lh.lh_validate(shp, lh.LH_BF16) == lh.LH_OK
        assert lh.lh_validate(shp, lh.LH_F32) == lh.LH_OK


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(d=32), dict(p=1), dict(L=0), dict(L=9), dict(N=4095),
    dict(S_=0), dict(S_=4096 + 1024 + 256 + 1), dict(B=0), dict(H=0), dict(N=0),
    dict(N=16, p=4, L=4),  # p^(L-1) = 64 > N
])
def test_validate_rejects_bad_shapes(bad):
    assert lh.lh_validate(S(**bad), lh.LH_BF16) == lh.LH_ERR_SHAPE


def test_validate_rejects_bad_dtype_and_null_shape():
    assert lh.lh_validate(S(), 7) == lh.LH_ERR_INVALID_ARG
    f = lh._lib().lh_validate
    assert f(None, lh.LH_BF16) == lh.LH_ERR_INVALID_ARG


def test_num_entries_and_sizes():
    shp = S(1, 16, 98304, 64, 4, 4, 8192)
    M = 98304 + 24576 + 6144 + 1536
    assert lh.lh_num_entries(shp) == M
    assert lh.lh_num_entries(S(d=96)) == -1
    saved = lh.lh_saved_bytes(shp)
    U = 16
    assert saved >= U * (8192 * 4 * 2 + M * 4 + 4 * 8192 * 64 * 2 + 8192 * 4 + 98304 * 4)
    offs = [lh.lh_saved_offset(shp, i) for i in range(9)]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert lh.lh_saved_offset(shp, 9) == -1
    ws_f = lh.lh_workspace_bytes(shp, lh.LH_BF16, False)
    ws_b = lh.lh_workspace_bytes(shp, lh.LH_BF16, True)
    assert ws_f >= U * (3 * (M - 98304) * 64 * 4 + M * 4)
    assert ws_b >= ws_f and ws_b >= U * 8192 * (64 * 2 + 4 + 3 * 64 * 4)
    assert lh.lh_workspace_bytes(S(d=96), lh.LH_BF16, True) == 0
    assert lh.lh_topk_workspace_bytes(shp) > 0  # the device-wide passes
    assert lh.lh_attn_bwd_workspace_bytes(shp) >= U * 8192 * 4


def test_bad_arguments_fail_before_any_launch():
    """Null/misaligned pointers and short workspaces return errors without a GPU."""
    lib = lh._lib()
    shp = S()
    r = lib.lh_forward(ctypes.byref(shp), lh.LH_BF16, None, None, None, 0.0, None, None, None,
                       0, None)
    assert r == lh.LH_ERR_INVALID_ARG
    p = 1 << 20  # a fake, aligned address: never dereferenced because the check fails first
    r = lib.lh_forward(ctypes.byref(shp), lh.LH_BF16, p, p, p, 0.0, p, p, p, 16, None)
    assert r == lh.LH_ERR_WORKSPACE
    r = lib.lh_score(ctypes.byref(shp), lh.LH_BF16, p + 4, p, p, None)
    assert r == lh.LH_ERR_INVALID_ARG
    r = lib.lh_subseq_attn_bwd(ctypes.byref(shp), p, p, p, p, p, p, 0.0, p, p, p, p, 0, None)
    assert r == lh.LH_ERR_WORKSPACE
    bad = S(d=96)
    r = lib.lh_gather(ctypes.byref(bad), lh.LH_BF16, p, p, p, p, p, p, p, p, p, p, None)
    assert r == lh.LH_ERR_SHAPE


def test_status_strings():
    for c in range(7):
        assert lh.lh_status_string(c).startswith("LH_")


def test_attention_impl_switch_roundtrip():
    prev = lh.lh_set_attention_impl(1)
    assert lh.lh_set_attention_impl(prev) == 1


def test_options_are_checked_on_the_host():
    """lh_options: NULL or zero is the default; keep_coarsest needs N/p^(L-1) <= S;
    modes and the reserved word are range-checked; the _ex calls reject bad
    options before any launch (and the same argument errors as the plain calls)."""
    lib = lh._lib()
    shp = S(1, 2, 4096, 64, 4, 4, 512)             # 64 coarsest entries <= 512
    assert lh.lh_validate_options(shp, None) == lh.LH_OK
    assert lh.lh_validate_options(shp, lh.make_options()) == lh.LH_OK
    for sm in (0, 1, 2):
        for cm in (0, 1, 2):
            assert lh.lh_validate_options(shp, lh.make_options(True, sm, cm)) == lh.LH_OK
    tight = S(1, 2, 4096, 64, 4, 2, 512)           # 1024 coarsest entries > 512
    assert lh.lh_validate_options(tight, lh.make_options(True)) == lh.LH_ERR_SHAPE
    assert lh.lh_validate_options(tight, lh.make_options(False)) == lh.LH_OK
    for bad in (lh.make_options(False, 3), lh.make_options(False, -1), lh.make_options(False, 0, 3)):
        assert lh.lh_validate_options(shp, bad) == lh.LH_ERR_INVALID_ARG
    o = lh.make_options()
    o.keep_coarsest = 2
    assert lh.lh_validate_options(shp, o) == lh.LH_ERR_INVALID_ARG
    o = lh.make_options()
    o.reserved = 1
    assert lh.lh_validate_options(shp, o) == lh.LH_ERR_INVALID_ARG
    assert lh.lh_validate_options(S(d=96), None) == lh.LH_ERR_SHAPE
    p = 1 << 20
    ob = ctypes.byref(lh.make_options(False, 5))
    assert lib.lh_forward_ex(ctypes.byref(shp), lh.LH_BF16, p, p, p, 0.0, p, p, p, 1 << 40, ob,
                             None) == lh.LH_ERR_INVALID_ARG
    assert lib.lh_topk_select_ex(ctypes.byref(tight), p, p, p, p, None, 0,
                                 ctypes.byref(lh.make_options(True)), None) == lh.LH_ERR_SHAPE
    assert lib.lh_backward_ex(ctypes.byref(shp), lh.LH_BF16, p, p, 0.0, p, p, p, p, 16,
                              None, None) == lh.LH_ERR_WORKSPACE
    assert lib.lh_scatter_back_ex(ctypes.byref(shp), lh.LH_BF16, p, p, p + 4, None, None,
                                  None) == lh.LH_ERR_INVALID_ARG


def test_forward_topk_path_rule():
    """lh_forward selects with the device-wide passes (faster than one cluster per
    unit at every benchmark shape once the passes are dependent launches)."""
    assert lh.lh_forward_topk_path(S(1, 16, 98304, 64, 4, 4, 8192)) == 1
    assert lh.lh_forward_topk_path(S(1, 16, 524288, 64, 4, 5, 16384)) == 1
    assert lh.lh_forward_topk_path(S(1, 8, 1048576, 128, 4, 6, 16384)) == 1
    assert lh.lh_forward_topk_path(S(d=96)) == -1


def test_forward_gather_path_rule():
    """lh_forward gathers through the pyramid for the benchmark workloads (their
    worst-case spans are far more rows than the levels) and pooled from the input
    for a small budget over a long input; invalid shapes give -1."""
    for shp in (S(1, 16, 98304, 64, 4, 4, 8192), S(1, 16, 524288, 64, 4, 5, 16384),
                S(1, 8, 1048576, 128, 4, 6, 16384), S()):
        assert lh.lh_forward_gather_path(shp, lh.LH_BF16) == 0
    assert lh.lh_forward_gather_path(S(1, 2, 65536, 64, 4, 3, 256), lh.LH_BF16) == 1
    assert lh.lh_forward_gather_path(S(1, 1, 100, 64, 2, 1, 100), lh.LH_BF16) == 0  # L = 1: no level
    assert lh.lh_forward_gather_path(S(d=96), lh.LH_BF16) == -1
