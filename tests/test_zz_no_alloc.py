"""lh_subseq_attn_bwd_noalloc: the attention backward without caller memory.

Some callers cannot allocate device memory or pass a workspace (a memory
planner owns every byte, or cudaMalloc is off limits mid-step because it can
synchronise the device).  This entry point keeps its scratch in a fixed array
inside the library instead.  It runs the same kernels as lh_subseq_attn_bwd on
the same inputs, so the GPU test calls it through the C ABI twice in a row and
requires both results to be bitwise equal to that call's (stricter than the
attention tolerance the other parity tests use).  This file is collected last
on purpose.
"""
import ctypes

import pytest
import torch

from long_context_lh_b200 import lighthouse as lh


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = lh._lib()
    shp = lh.make_shape(1, 256, 8192, 64, 2, 1, 8192)  # 2,097,152 rows > 1,048,576
    p = 1 << 20  # aligned fake address, never dereferenced: the size check comes first
    r = lib.lh_subseq_attn_bwd_noalloc(ctypes.byref(shp), p, p, p, p, p, p, 0.0, p, p, p, None)
    assert r == lh.LH_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("U,S,d", [(16, 1024, 64), (3, 777, 128)])
def test_noalloc_matches_workspace_entry_point_twice(U, S, d):
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev).manual_seed(4242 + S)
    qs, ks, vs, dos = (torch.randn((1, U, S, d), generator=g, device=dev).to(torch.float16)
                       for _ in range(4))
    shp = lh.make_shape(1, U, S, d, 2, 1, S)
    os_ = torch.empty_like(qs)
    lse = torch.empty((1, U, S), dtype=torch.float32, device=dev)
    lh.lh_subseq_attn_fwd(shp, qs, ks, vs, 0.0, os_, lse)
    ref = [torch.empty((1, U, S, d), dtype=torch.float32, device=dev) for _ in range(3)]
    wsb = lh.lh_attn_bwd_workspace_bytes(shp)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    lh.lh_subseq_attn_bwd(shp, qs, ks, vs, os_, lse, dos, 0.0, *ref, ws, wsb)
    for call in range(2):
        got = [torch.full((1, U, S, d), float("nan"), device=dev) for _ in range(3)]
        lh.lh_subseq_attn_bwd_noalloc(shp, qs, ks, vs, os_, lse, dos, 0.0, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("dqs", "dks", "dvs"), got, ref):
            assert torch.equal(a, b), f"call {call} {name}: differs from lh_subseq_attn_bwd"
