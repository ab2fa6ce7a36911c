"""Thin ctypes binding of liblighthouse.so (include/lighthouse.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Functions keep the C names; tensors are torch tensors on the GPU
(contiguous, row-major), streams default to torch's current stream.  If the
library is missing this module raises on first use: there is no fallback.

`forward`/`backward` below are conveniences that allocate the outputs, the
saved state and the workspace with torch and call lh_forward / lh_backward.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# LH_LIBRARY=debug selects the bounds-checking build (liblighthouse_debug.so):
# the same entry points, with every data-dependent index checked in the kernels
# and failures reported through lh_read_device_status.
LIB_PATH = os.path.join(
    _PKG, "liblighthouse_debug.so" if os.environ.get("LH_LIBRARY") == "debug" else "liblighthouse.so")

LH_OK, LH_ERR_INVALID_ARG, LH_ERR_SHAPE, LH_ERR_UNSUPPORTED = 0, 1, 2, 3
LH_ERR_WORKSPACE, LH_ERR_CUDA, LH_ERR_DEVICE_STATUS = 4, 5, 6
LH_F32, LH_BF16 = 0, 1
# bits of the device status word (lh_read_device_status)
LH_STATUS_ATTN_FWD_TIMEOUT, LH_STATUS_ATTN_BWD_TIMEOUT, LH_STATUS_FP16_SATURATED = 0x100, 0x200, 0x400
LH_STATUS_BOUNDS = 0x800  # debug build only

SAVED_IDX, SAVED_POS, SAVED_SLOT, SAVED_QS, SAVED_KS, SAVED_VS, SAVED_OS, SAVED_LSE, \
    SAVED_INV_COUNT = range(9)


class LighthouseError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = _lib().lh_status_string(code).decode()
        super().__init__(f"{fn}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64),
                ("d", ctypes.c_int32), ("p", ctypes.c_int32), ("L", ctypes.c_int32),
                ("S", ctypes.c_int32)]

    def __repr__(self):
        return (f"Shape(B={self.B}, H={self.H}, N={self.N}, d={self.d}, p={self.p}, "
                f"L={self.L}, S={self.S})")


def make_shape(B, H, N, d, p, L, S) -> Shape:
    return Shape(int(B), int(H), int(N), int(d), int(p), int(L), int(S))


LH_SCORE_SUM, LH_SCORE_PRODUCT, LH_SCORE_CONCAT = 0, 1, 2
LH_SCATTER_MEAN, LH_SCATTER_SUM, LH_SCATTER_LAST = 0, 1, 2


class Options(ctypes.Structure):
    """lh_options: layer variants (keep-coarsest-level, score and scatter ablations)."""
    _fields_ = [("keep_coarsest", ctypes.c_int32), ("score_mode", ctypes.c_int32),
                ("scatter_mode", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def make_options(keep_coarsest=False, score_mode=LH_SCORE_SUM,
                 scatter_mode=LH_SCATTER_MEAN) -> Options:
    o = Options()
    o.keep_coarsest = 1 if keep_coarsest else 0
    o.score_mode = int(score_mode)
    o.scatter_mode = int(scatter_mode)
    return o


def _opt(options):
    return None if options is None else ctypes.byref(options)


_VP = ctypes.c_void_p
_SP = ctypes.POINTER(Shape)
_I, _F, _SZ, _I64 = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64
_SIGS = {
    "lh_status_string": ([_I], ctypes.c_char_p),
    "lh_validate": ([_SP, _I], _I),
    "lh_num_entries": ([_SP], _I64),
    "lh_workspace_bytes": ([_SP, _I, _I], _SZ),
    "lh_saved_bytes": ([_SP], _SZ),
    "lh_saved_offset": ([_SP, _I], _I64),
    "lh_build_pyramid": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_build_pyramid_score": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_score": ([_SP, _I, _VP, _VP, _VP, _VP], _I),
    "lh_topk_workspace_bytes": ([_SP], _SZ),
    "lh_forward_topk_path": ([_SP], _I),
    "lh_topk_select": ([_SP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP], _I),
    "lh_gather": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_gather_pooled": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_subseq_attn_fwd": ([_SP, _VP, _VP, _VP, _F, _VP, _VP, _VP], _I),
    "lh_attn_bwd_workspace_bytes": ([_SP], _SZ),
    "lh_subseq_attn_bwd": ([_SP, _VP, _VP, _VP, _VP, _VP, _VP, _F, _VP, _VP, _VP, _VP, _SZ,
                            _VP], _I),
    "lh_subseq_attn_bwd_noalloc": ([_SP, _VP, _VP, _VP, _VP, _VP, _VP, _F, _VP, _VP, _VP,
                                    _VP], _I),
    "lh_block_attn_fwd": ([_SP, _I, _VP, _VP, _VP, _F, _VP, _VP, _VP], _I),
    "lh_block_attn_merge": ([_I64, _I, _VP, _VP, _VP, _VP, _I, _VP], _I),
    "lh_block_attn_finish": ([_I64, _I, _VP, _VP, _VP], _I),
    "lh_block_attn_bwd": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _F, _VP, _VP, _VP, _VP, _SZ,
                           _VP], _I),
    "lh_accumulate": ([_I64, _VP, _VP, _VP], _I),
    "lh_forward_gather_path": ([_SP, _I], _I),
    "lh_scatter_back": ([_SP, _I, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_scatter_back_bwd": ([_SP, _I, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_gather_bwd": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_forward": ([_SP, _I, _VP, _VP, _VP, _F, _VP, _VP, _VP, _SZ, _VP], _I),
    "lh_backward": ([_SP, _I, _VP, _VP, _F, _VP, _VP, _VP, _VP, _SZ, _VP], _I),
    "lh_read_device_status": ([_VP, ctypes.POINTER(ctypes.c_uint32)], _I),
    "lh_set_attention_impl": ([_I], _I),
    "lh_validate_options": ([_SP, _VP], _I),
    "lh_build_pyramid_score_ex": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_score_ex": ([_SP, _I, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_topk_select_ex": ([_SP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP], _I),
    "lh_forward_ex": ([_SP, _I, _VP, _VP, _VP, _F, _VP, _VP, _VP, _SZ, _VP, _VP], _I),
    "lh_backward_ex": ([_SP, _I, _VP, _VP, _F, _VP, _VP, _VP, _VP, _SZ, _VP, _VP], _I),
    "lh_scatter_back_ex": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_scatter_back_bwd_ex": ([_SP, _I, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "lh_attention_impl_in_use": ([], _I),
    "lh_kernel_launches": ([_SP, _I, _I], _I),
}
EXPORTED = tuple(_SIGS)

_L = None


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_lh_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _L = lib
    return _L


def _check(fn: str, code: int):
    if code != LH_OK:
        raise LighthouseError(fn, code)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _st(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return LH_BF16
    if t == torch.float32:
        return LH_F32
    raise ValueError(f"unsupported dtype {t}")


# --------------------------------------------------------------- queries
def lh_validate(shape: Shape, dtype: int) -> int:
    return _lib().lh_validate(ctypes.byref(shape), dtype)


def lh_num_entries(shape: Shape) -> int:
    return int(_lib().lh_num_entries(ctypes.byref(shape)))


def lh_workspace_bytes(shape: Shape, dtype: int, with_backward: bool) -> int:
    return int(_lib().lh_workspace_bytes(ctypes.byref(shape), dtype, int(with_backward)))


def lh_saved_bytes(shape: Shape) -> int:
    return int(_lib().lh_saved_bytes(ctypes.byref(shape)))


def lh_saved_offset(shape: Shape, which: int) -> int:
    return int(_lib().lh_saved_offset(ctypes.byref(shape), which))


def lh_topk_workspace_bytes(shape: Shape) -> int:
    return int(_lib().lh_topk_workspace_bytes(ctypes.byref(shape)))


def lh_forward_topk_path(shape: Shape) -> int:
    return int(_lib().lh_forward_topk_path(ctypes.byref(shape)))


def lh_attn_bwd_workspace_bytes(shape: Shape) -> int:
    return int(_lib().lh_attn_bwd_workspace_bytes(ctypes.byref(shape)))


def lh_status_string(code: int) -> str:
    return _lib().lh_status_string(code).decode()


def lh_set_attention_impl(impl: int) -> int:
    return int(_lib().lh_set_attention_impl(impl))


def lh_attention_impl_in_use() -> int:
    return int(_lib().lh_attention_impl_in_use())


def lh_forward_gather_path(shape: Shape, dtype: int) -> int:
    return int(_lib().lh_forward_gather_path(ctypes.byref(shape), int(dtype)))


def lh_kernel_launches(shape: Shape, dtype: int, backward: bool) -> int:
    return int(_lib().lh_kernel_launches(ctypes.byref(shape), int(dtype), int(backward)))


def lh_read_device_status(stream=None) -> int:
    code = ctypes.c_uint32(0)
    r = _lib().lh_read_device_status(_st(stream), ctypes.byref(code))
    if r not in (LH_OK, LH_ERR_DEVICE_STATUS):
        _check("lh_read_device_status", r)
    return int(code.value)


# ---------------------------------------------------------------- stages
def lh_build_pyramid(shape, dtype, q, k, v, pq, pk, pv, stream=None):
    _check("lh_build_pyramid", _lib().lh_build_pyramid(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _st(stream)))


def lh_build_pyramid_score(shape, dtype, q, k, v, pq, pk, pv, score, stream=None):
    _check("lh_build_pyramid_score", _lib().lh_build_pyramid_score(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _p(score),
        _st(stream)))


def lh_validate_options(shape, options):
    return _lib().lh_validate_options(ctypes.byref(shape), _opt(options))


def lh_build_pyramid_score_ex(shape, dtype, q, k, v, pq, pk, pv, score, options, stream=None):
    _check("lh_build_pyramid_score_ex", _lib().lh_build_pyramid_score_ex(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _p(score),
        _opt(options), _st(stream)))


def lh_score_ex(shape, dtype, q, k, score, options, stream=None):
    _check("lh_score_ex", _lib().lh_score_ex(ctypes.byref(shape), dtype, _p(q), _p(k), _p(score),
                                             _opt(options), _st(stream)))


def lh_topk_select_ex(shape, score, idx, pos, slot, options, ws=None, ws_bytes=0, stream=None):
    _check("lh_topk_select_ex", _lib().lh_topk_select_ex(
        ctypes.byref(shape), _p(score), _p(idx), _p(pos), _p(slot), _p(ws), ws_bytes,
        _opt(options), _st(stream)))


def lh_forward_ex(shape, dtype, q, k, v, scale, o, saved, ws, ws_bytes, options, stream=None):
    _check("lh_forward_ex", _lib().lh_forward_ex(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), float(scale), _p(o), _p(saved), _p(ws),
        ws_bytes, _opt(options), _st(stream)))


def lh_backward_ex(shape, dtype, saved, dO, scale, dq, dk, dv, ws, ws_bytes, options, stream=None):
    _check("lh_backward_ex", _lib().lh_backward_ex(
        ctypes.byref(shape), dtype, _p(saved), _p(dO), float(scale), _p(dq), _p(dk), _p(dv),
        _p(ws), ws_bytes, _opt(options), _st(stream)))


def lh_scatter_back_ex(shape, dtype, os_, slot, o, inv_count, options, stream=None):
    _check("lh_scatter_back_ex", _lib().lh_scatter_back_ex(
        ctypes.byref(shape), dtype, _p(os_), _p(slot), _p(o), _p(inv_count), _opt(options),
        _st(stream)))


def lh_scatter_back_bwd_ex(shape, dtype, dO, slot, inv_count, dos, options, stream=None):
    _check("lh_scatter_back_bwd_ex", _lib().lh_scatter_back_bwd_ex(
        ctypes.byref(shape), dtype, _p(dO), _p(slot), _p(inv_count), _p(dos), _opt(options),
        _st(stream)))


def lh_score(shape, dtype, q, k, score, stream=None):
    _check("lh_score", _lib().lh_score(ctypes.byref(shape), dtype, _p(q), _p(k), _p(score),
                                       _st(stream)))


def lh_topk_select(shape, score, idx, pos, slot, ws=None, ws_bytes=0, stream=None):
    _check("lh_topk_select", _lib().lh_topk_select(
        ctypes.byref(shape), _p(score), _p(idx), _p(pos), _p(slot), _p(ws), ws_bytes,
        _st(stream)))


def lh_gather(shape, dtype, q, k, v, pq, pk, pv, idx, qs, ks, vs, stream=None):
    _check("lh_gather", _lib().lh_gather(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _p(idx),
        _p(qs), _p(ks), _p(vs), _st(stream)))


def lh_gather_pooled(shape, dtype, q, k, v, idx, qs, ks, vs, stream=None):
    _check("lh_gather_pooled", _lib().lh_gather_pooled(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), _p(idx), _p(qs), _p(ks), _p(vs),
        _st(stream)))


def lh_subseq_attn_fwd(shape, qs, ks, vs, scale, os_, lse, stream=None):
    _check("lh_subseq_attn_fwd", _lib().lh_subseq_attn_fwd(
        ctypes.byref(shape), _p(qs), _p(ks), _p(vs), float(scale), _p(os_), _p(lse),
        _st(stream)))


def lh_subseq_attn_bwd(shape, qs, ks, vs, os_, lse, dos, scale, dqs, dks, dvs, ws, ws_bytes,
                       stream=None):
    _check("lh_subseq_attn_bwd", _lib().lh_subseq_attn_bwd(
        ctypes.byref(shape), _p(qs), _p(ks), _p(vs), _p(os_), _p(lse), _p(dos), float(scale),
        _p(dqs), _p(dks), _p(dvs), _p(ws), ws_bytes, _st(stream)))


def lh_subseq_attn_bwd_noalloc(shape, qs, ks, vs, os_, lse, dos, scale, dqs, dks, dvs,
                               stream=None):
    _check("lh_subseq_attn_bwd_noalloc", _lib().lh_subseq_attn_bwd_noalloc(
        ctypes.byref(shape), _p(qs), _p(ks), _p(vs), _p(os_), _p(lse), _p(dos), float(scale),
        _p(dqs), _p(dks), _p(dvs), _st(stream)))


# ------------------------------------------------ context parallelism (one GPU's ring steps)
def lh_block_attn_fwd(shape, causal, qs, ks, vs, scale, os_, lse, stream=None):
    _check("lh_block_attn_fwd", _lib().lh_block_attn_fwd(
        ctypes.byref(shape), int(causal), _p(qs), _p(ks), _p(vs), float(scale), _p(os_), _p(lse),
        _st(stream)))


def lh_block_attn_merge(rows, d, o_acc, lse_acc, o_part, lse_part, first, stream=None):
    _check("lh_block_attn_merge", _lib().lh_block_attn_merge(
        int(rows), int(d), _p(o_acc), _p(lse_acc), _p(o_part), _p(lse_part), int(first), _st(stream)))


def lh_block_attn_finish(rows, d, o_acc, os_, stream=None):
    _check("lh_block_attn_finish", _lib().lh_block_attn_finish(int(rows), int(d), _p(o_acc), _p(os_),
                                                               _st(stream)))


def lh_block_attn_bwd(shape, causal, qs, ks, vs, os_, lse, dos, scale, dqs, dks, dvs, ws, ws_bytes,
                      stream=None):
    _check("lh_block_attn_bwd", _lib().lh_block_attn_bwd(
        ctypes.byref(shape), int(causal), _p(qs), _p(ks), _p(vs), _p(os_), _p(lse), _p(dos),
        float(scale), _p(dqs), _p(dks), _p(dvs), _p(ws), int(ws_bytes), _st(stream)))


def lh_accumulate(n, acc, x, stream=None):
    _check("lh_accumulate", _lib().lh_accumulate(int(n), _p(acc), _p(x), _st(stream)))


def lh_scatter_back(shape, dtype, os_, slot, o, inv_count=None, stream=None):
    _check("lh_scatter_back", _lib().lh_scatter_back(
        ctypes.byref(shape), dtype, _p(os_), _p(slot), _p(o), _p(inv_count), _st(stream)))


def lh_scatter_back_bwd(shape, dtype, dO, slot, inv_count, dos, stream=None):
    _check("lh_scatter_back_bwd", _lib().lh_scatter_back_bwd(
        ctypes.byref(shape), dtype, _p(dO), _p(slot), _p(inv_count), _p(dos), _st(stream)))


def lh_gather_bwd(shape, dtype, dqs, dks, dvs, slot, dq, dk, dv, stream=None):
    _check("lh_gather_bwd", _lib().lh_gather_bwd(
        ctypes.byref(shape), dtype, _p(dqs), _p(dks), _p(dvs), _p(slot), _p(dq), _p(dk), _p(dv),
        _st(stream)))


def lh_forward(shape, dtype, q, k, v, scale, o, saved, ws, ws_bytes, stream=None):
    _check("lh_forward", _lib().lh_forward(
        ctypes.byref(shape), dtype, _p(q), _p(k), _p(v), float(scale), _p(o), _p(saved), _p(ws),
        ws_bytes, _st(stream)))


def lh_backward(shape, dtype, saved, dO, scale, dq, dk, dv, ws, ws_bytes, stream=None):
    _check("lh_backward", _lib().lh_backward(
        ctypes.byref(shape), dtype, _p(saved), _p(dO), float(scale), _p(dq), _p(dk), _p(dv),
        _p(ws), ws_bytes, _st(stream)))


# ---------------------------------------------------------- conveniences
def saved_view(shape: Shape, saved: torch.Tensor, which: int) -> torch.Tensor:
    """A typed view of one region of the saved buffer (idx, pos, slot, qs, ...)."""
    S, d, N = shape.S, shape.d, shape.N
    M = lh_num_entries(shape)
    off = lh_saved_offset(shape, which)
    spec = {SAVED_IDX: (torch.int32, (shape.B, shape.H, S)),
            SAVED_POS: (torch.int32, (shape.B, shape.H, S)),
            SAVED_SLOT: (torch.int32, (shape.B, shape.H, M)),
            SAVED_QS: (torch.float16, (shape.B, shape.H, S, d)),
            SAVED_KS: (torch.float16, (shape.B, shape.H, S, d)),
            SAVED_VS: (torch.float16, (shape.B, shape.H, S, d)),
            SAVED_OS: (torch.float16, (shape.B, shape.H, S, d)),
            SAVED_LSE: (torch.float32, (shape.B, shape.H, S)),
            SAVED_INV_COUNT: (torch.float32, (shape.B, shape.H, N))}[which]
    dt, shp = spec
    n = 1
    for x in shp:
        n *= x
    nbytes = n * torch.tensor([], dtype=dt).element_size()
    return saved[off:off + nbytes].view(dt).view(shp)


@dataclass
class Saved:
    shape: Shape
    dtype: int
    scale: float
    buf: torch.Tensor
    options: object = None  # the Options lh_forward_ex got (the backward needs them too)


def forward(q, k, v, p: int, L: int, S: int, scale: float = 0.0, stream=None, options=None):
    """o, Saved = forward(q, k, v, p, L, S): whole layer through lh_forward
    (lh_forward_ex when `options`, an Options, is given)."""
    B, H, N, d = q.shape
    shp = make_shape(B, H, N, d, p, L, S)
    dt = dtype_code(q.dtype)
    _check("lh_validate", lh_validate(shp, dt))
    _check("lh_validate_options", lh_validate_options(shp, options))
    o = torch.empty_like(q)
    saved = torch.empty(lh_saved_bytes(shp), dtype=torch.uint8, device=q.device)
    wsb = lh_workspace_bytes(shp, dt, False)
    ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=q.device)
    if options is None:
        lh_forward(shp, dt, q, k, v, scale, o, saved, ws, wsb, stream)
    else:
        lh_forward_ex(shp, dt, q, k, v, scale, o, saved, ws, wsb, options, stream)
    return o, Saved(shp, dt, scale, saved, options)


def backward(saved: Saved, dO, stream=None):
    """dq, dk, dv = backward(saved, dO): whole backward through lh_backward."""
    shp, dt = saved.shape, saved.dtype
    dq, dk, dv = (torch.empty_like(dO) for _ in range(3))
    wsb = lh_workspace_bytes(shp, dt, True)
    ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dO.device)
    if saved.options is None:
        lh_backward(shp, dt, saved.buf, dO, saved.scale, dq, dk, dv, ws, wsb, stream)
    else:
        lh_backward_ex(shp, dt, saved.buf, dO, saved.scale, dq, dk, dv, ws, wsb, saved.options,
                       stream)
    return dq, dk, dv


class LighthouseAttention(torch.autograd.Function):
    """autograd wrapper: y = LighthouseAttention.apply(q, k, v, p, L, S, scale, options)."""

    @staticmethod
    def forward(ctx, q, k, v, p, L, S, scale=0.0, options=None):
        o, saved = forward(q.contiguous(), k.contiguous(), v.contiguous(), p, L, S, scale,
                           options=options)
        ctx.saved_state = saved
        return o

    @staticmethod
    def backward(ctx, dO):
        dq, dk, dv = backward(ctx.saved_state, dO.contiguous())
        return dq, dk, dv, None, None, None, None, None
