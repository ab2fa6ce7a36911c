"""CPU oracle for one Lighthouse Attention layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never does, and this package never imports the product.

The arithmetic lives in ``lh_oracle.c`` (plain C, POSIX threads); this module
only builds it with gcc, loads it with ctypes and marshals numpy arrays.  The
pipeline helpers at the bottom compose the stages in the order the pages give
them (pyramid -> score -> joint top-K -> gather -> attention -> scatter-back,
and the backward through scatter-back, attention and gather).

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against something other than itself (closed forms, brute force, torch's SDPA in
fp64, finite differences, adjoint identities, a hand-worked example).  The
choice of how the two norms combine (their sum) and of how a coarse output
spreads over its span (mean over contributors) are readings of the pages that
no page value can confirm: for those two choices parity is unpinned against
the pages themselves (the arithmetic under each reading is pinned).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lh_oracle.c")
_LIB = os.path.join(_HERE, "liblh_oracle.so")


def build(force: bool = False) -> str:
    """Compile lh_oracle.c into liblh_oracle.so next to it (gcc, -O2, no fp contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("N", ctypes.c_int64),
                ("d", ctypes.c_int32), ("p", ctypes.c_int32), ("L", ctypes.c_int32),
                ("S", ctypes.c_int32)]


@dataclass(frozen=True)
class Shape:
    B: int
    H: int
    N: int
    d: int
    p: int
    L: int
    S: int

    @property
    def U(self) -> int:
        return self.B * self.H

    def level_len(self, l: int) -> int:
        return self.N // self.p ** l

    def level_off(self, l: int) -> int:
        return sum(self.level_len(m) for m in range(l))

    @property
    def M(self) -> int:
        return self.level_off(self.L)

    def c(self) -> _Shape:
        return _Shape(self.B, self.H, self.N, self.d, self.p, self.L, self.S)

    def unit(self) -> "Shape":
        """The same problem restricted to one (b, h) unit."""
        return Shape(1, 1, self.N, self.d, self.p, self.L, self.S)


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        sp = ctypes.POINTER(_Shape)
        i = ctypes.c_int
        i64 = ctypes.c_int64
        d = ctypes.c_double
        sig = {
            "lho_num_entries": ([sp], i64),
            "lho_pyramid": ([sp, P, P, i], None),
            "lho_score": ([sp, P, P, P, i], None),
            "lho_select": ([sp, P, P, P, P, i], None),
            "lho_score_mode": ([sp, P, P, P, i, i], None),
            "lho_select_opt": ([sp, P, P, P, P, i, i], None),
            "lho_gather": ([sp, P, P, P, P], None),
            "lho_attn_fwd": ([sp, P, P, P, d, P, i64, P, P, i], None),
            "lho_attn_bwd": ([sp, P, P, P, P, d, P, P, P, i], None),
            "lho_scatter": ([sp, P, P, P], None),
            "lho_scatter_bwd": ([sp, P, P, P, P], None),
            "lho_scatter_mode": ([sp, P, P, P, i], None),
            "lho_scatter_bwd_mode": ([sp, P, P, P, P, i], None),
            "lho_gather_bwd": ([sp, P, P, P], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(_lib, name)
            f.argtypes = args
            f.restype = res
    return _lib


def _threads(nthreads):
    return int(nthreads) if nthreads else (os.cpu_count() or 1)


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


# ----------------------------------------------------------------- stages
def num_entries(s: Shape) -> int:
    return int(_L().lho_num_entries(ctypes.byref(s.c())))


def pyramid(s: Shape, x, nthreads=None) -> np.ndarray:
    """Levels 1..L-1 of the average-pooling pyramid, fp64 [B,H,M-N,d]."""
    x = _f64(x).reshape(s.U, s.N, s.d)
    out = np.zeros((s.U, s.M - s.N, s.d), np.float64)
    _L().lho_pyramid(ctypes.byref(s.c()), _p(x), _p(out), _threads(nthreads))
    return out.reshape(s.B, s.H, s.M - s.N, s.d)


SCORE_SUM, SCORE_PRODUCT, SCORE_CONCAT = 0, 1, 2  # how the two level-0 norms combine


def score(s: Shape, q, k, nthreads=None, mode=SCORE_SUM) -> np.ndarray:
    """fp32 scores of all M entries [B,H,M] (at level 0 the norm sum, or the
    ablations: norm product, norm of [q; k]; max-pool above)."""
    q = _f32(q).reshape(s.U, s.N, s.d)
    k = _f32(k).reshape(s.U, s.N, s.d)
    out = np.zeros((s.U, s.M), np.float32)
    _L().lho_score_mode(ctypes.byref(s.c()), _p(q), _p(k), _p(out), int(mode), _threads(nthreads))
    return out.reshape(s.B, s.H, s.M)


def select(s: Shape, sc, nthreads=None, keep_coarsest=False):
    """Joint top-S by (score desc, gid asc), ordered by (pos asc, level asc);
    keep_coarsest ranks every level-(L-1) entry above every score.

    Returns idx [B,H,S] (gid), pos [B,H,S], slot [B,H,M] (slot or -1)."""
    sc = _f32(sc).reshape(s.U, s.M)
    idx = np.zeros((s.U, s.S), np.int32)
    pos = np.zeros((s.U, s.S), np.int32)
    slot = np.zeros((s.U, s.M), np.int32)
    _L().lho_select_opt(ctypes.byref(s.c()), _p(sc), _p(idx), _p(pos), _p(slot),
                        1 if keep_coarsest else 0, _threads(nthreads))
    return (idx.reshape(s.B, s.H, s.S), pos.reshape(s.B, s.H, s.S),
            slot.reshape(s.B, s.H, s.M))


def gather(s: Shape, x, pyr, idx) -> np.ndarray:
    x = _f64(x).reshape(s.U, s.N, s.d)
    pyr = _f64(pyr).reshape(s.U, s.M - s.N, s.d)
    idx = _i32(idx).reshape(s.U, s.S)
    out = np.zeros((s.U, s.S, s.d), np.float64)
    _L().lho_gather(ctypes.byref(s.c()), _p(x), _p(pyr), _p(idx), _p(out))
    return out.reshape(s.B, s.H, s.S, s.d)


def attn_fwd(s: Shape, qs, ks, vs, scale, rows=None, nthreads=None):
    """Causal attention over the slot index; returns (os, lse) for `rows` (all if None)."""
    qs, ks, vs = (_f64(t).reshape(s.U, s.S, s.d) for t in (qs, ks, vs))
    if rows is None:
        nrows, rp = s.S, None
    else:
        rows = _i32(rows)
        nrows, rp = rows.size, _p(rows)
    os_ = np.zeros((s.U, nrows, s.d), np.float64)
    lse = np.zeros((s.U, nrows), np.float64)
    _L().lho_attn_fwd(ctypes.byref(s.c()), _p(qs), _p(ks), _p(vs), float(scale), rp, nrows,
                      _p(os_), _p(lse), _threads(nthreads))
    return os_.reshape(s.B, s.H, nrows, s.d), lse.reshape(s.B, s.H, nrows)


def attn_bwd(s: Shape, qs, ks, vs, dos, scale, nthreads=None):
    qs, ks, vs, dos = (_f64(t).reshape(s.U, s.S, s.d) for t in (qs, ks, vs, dos))
    dq, dk, dv = (np.zeros((s.U, s.S, s.d), np.float64) for _ in range(3))
    _L().lho_attn_bwd(ctypes.byref(s.c()), _p(qs), _p(ks), _p(vs), _p(dos), float(scale),
                      _p(dq), _p(dk), _p(dv), _threads(nthreads))
    shp = (s.B, s.H, s.S, s.d)
    return dq.reshape(shp), dk.reshape(shp), dv.reshape(shp)


def attn_bwd_sampled(qs, ks, vs, dos, scale, rows, chunk=1024):
    """Gradients of causal softmax attention (one unit, fp64 numpy) at sampled
    positions, for sub-sequences too long for the full O(S^2 d) loops above.

    The softmax adjoint is separable: with P = softmax over k' <= k of
    scale * q_k . k_k', O = P V, D_k = dO_k . O_k and dS = P * (dO V^T - D),
      dQ[k]  = scale * sum_k' dS[k, k'] K[k']        (row k of dS),
      dK[k'] = scale * sum_k  dS[k, k'] Q[k]         (column k' of dS),
      dV[k'] = sum_k P[k, k'] dO[k]                  (column k' of P),
    ([ES] gist.science/es "Resumen Técnico: Pre-entrenamiento con Contexto
    Largo mediante Atención Lighthouse", §2.B: the backward through the dense
    sub-sequence attention is the stock one).  Row k needs every key; column
    k' needs every query's LSE and D, which one blocked pass over all rows of
    P gives.  Inputs [S, d]; returns dq[rows], dk[rows], dv[rows], [len(rows), d].
    """
    q, k, v, do = (np.asarray(t, np.float64) for t in (qs, ks, vs, dos))
    S = q.shape[0]
    rows = np.asarray(rows, np.int64)
    lse = np.empty(S)
    o = np.empty_like(q)
    for a in range(0, S, chunk):  # LSE and O of every row, blocked over rows
        b = min(S, a + chunk)
        z = scale * (q[a:b] @ k.T)
        z[np.arange(S)[None, :] > np.arange(a, b)[:, None]] = -np.inf  # key after the query
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        ssum = e.sum(axis=1, keepdims=True)
        lse[a:b] = (m + np.log(ssum))[:, 0]
        o[a:b] = (e / ssum) @ v
    dsum = np.einsum("kd,kd->k", do, o)  # D_k
    # rows of dS -> dQ
    zr = scale * (q[rows] @ k.T)
    keep = np.arange(S)[None, :] <= rows[:, None]
    pr = np.where(keep, np.exp(zr - lse[rows, None]), 0.0)
    dsr = pr * ((do[rows] @ v.T) - dsum[rows, None])
    dq = scale * (dsr @ k)
    # columns of P and dS -> dV, dK
    zc = scale * (q @ k[rows].T)  # [S, len(rows)]
    keepc = np.arange(S)[:, None] >= rows[None, :]
    pc = np.where(keepc, np.exp(zc - lse[:, None]), 0.0)
    dv = pc.T @ do
    dsc = pc * ((do @ v[rows].T) - dsum[:, None])
    dk = scale * (dsc.T @ q)
    return dq, dk, dv


SCATTER_MEAN, SCATTER_SUM, SCATTER_LAST = 0, 1, 2  # how a coarse output spreads over its span


def scatter(s: Shape, os_, slot, mode=SCATTER_MEAN) -> np.ndarray:
    """Scatter-back: the mean over a token's contributors (or the ablations: their
    sum; last-token-only delivery)."""
    os_ = _f64(os_).reshape(s.U, s.S, s.d)
    slot = _i32(slot).reshape(s.U, s.M)
    out = np.zeros((s.U, s.N, s.d), np.float64)
    _L().lho_scatter_mode(ctypes.byref(s.c()), _p(os_), _p(slot), _p(out), int(mode))
    return out.reshape(s.B, s.H, s.N, s.d)


def scatter_bwd(s: Shape, dO, idx, slot, mode=SCATTER_MEAN) -> np.ndarray:
    dO = _f64(dO).reshape(s.U, s.N, s.d)
    idx = _i32(idx).reshape(s.U, s.S)
    slot = _i32(slot).reshape(s.U, s.M)
    out = np.zeros((s.U, s.S, s.d), np.float64)
    _L().lho_scatter_bwd_mode(ctypes.byref(s.c()), _p(dO), _p(idx), _p(slot), _p(out), int(mode))
    return out.reshape(s.B, s.H, s.S, s.d)


def gather_bwd(s: Shape, dxs, slot) -> np.ndarray:
    dxs = _f64(dxs).reshape(s.U, s.S, s.d)
    slot = _i32(slot).reshape(s.U, s.M)
    out = np.zeros((s.U, s.N, s.d), np.float64)
    _L().lho_gather_bwd(ctypes.byref(s.c()), _p(dxs), _p(slot), _p(out))
    return out.reshape(s.B, s.H, s.N, s.d)


# --------------------------------------------------------------- pipeline
def default_scale(s: Shape, scale=None) -> float:
    return 1.0 / float(np.sqrt(s.d)) if (scale is None or scale <= 0) else float(scale)


def forward(s: Shape, q, k, v, scale=None, nthreads=None, score_mode=SCORE_SUM,
            keep_coarsest=False, scatter_mode=SCATTER_MEAN) -> dict:
    """The whole forward; returns every intermediate (fp64 except score)."""
    scale = default_scale(s, scale)
    pq, pk, pv = (pyramid(s, x, nthreads) for x in (q, k, v))
    sc = score(s, q, k, nthreads, mode=score_mode)
    idx, pos, slot = select(s, sc, nthreads, keep_coarsest=keep_coarsest)
    qs, ks, vs = gather(s, q, pq, idx), gather(s, k, pk, idx), gather(s, v, pv, idx)
    os_, lse = attn_fwd(s, qs, ks, vs, scale, nthreads=nthreads)
    o = scatter(s, os_, slot, scatter_mode)
    return dict(pq=pq, pk=pk, pv=pv, score=sc, idx=idx, pos=pos, slot=slot, qs=qs, ks=ks,
                vs=vs, os=os_, lse=lse, o=o, scale=scale, scatter_mode=scatter_mode)


def backward(s: Shape, fwd: dict, dO, nthreads=None) -> dict:
    """Backward through scatter-back, attention and gather with the saved selection."""
    dos = scatter_bwd(s, dO, fwd["idx"], fwd["slot"], fwd.get("scatter_mode", SCATTER_MEAN))
    dqs, dks, dvs = attn_bwd(s, fwd["qs"], fwd["ks"], fwd["vs"], dos, fwd["scale"], nthreads)
    return dict(dos=dos, dqs=dqs, dks=dks, dvs=dvs,
                dq=gather_bwd(s, dqs, fwd["slot"]), dk=gather_bwd(s, dks, fwd["slot"]),
                dv=gather_bwd(s, dvs, fwd["slot"]))


def forward_fixed(s: Shape, q, k, v, idx, slot, scale=None, nthreads=None) -> np.ndarray:
    """Forward with a frozen selection (used for finite differences)."""
    scale = default_scale(s, scale)
    xs = [gather(s, x, pyramid(s, x, nthreads), idx) for x in (q, k, v)]
    os_, _ = attn_fwd(s, *xs, scale, nthreads=nthreads)
    return scatter(s, os_, slot)


# ------------------------------------------------------- context parallelism
def cp_shards(s: Shape, P: int) -> Shape:
    """The per-shard shape of P-way context parallelism: N/P tokens, S/P entries."""
    if P < 1 or s.N % P or s.S % P:
        raise ValueError("N and S must be multiples of the shard count")
    return Shape(s.B, s.H, s.N // P, s.d, s.p, s.L, s.S // P)


def cp_forward(s: Shape, q, k, v, P: int, scale=None) -> dict:
    """The layer under P-way context parallelism ([PT] bitsgeniais.com.br, section
    "Escalando para o Céu (ou 1 Milhão de Tokens!): Paralelismo de Contexto"):
    the sequence is cut into P contiguous shards; each shard builds its own
    pyramid, scores and selection with a budget of S/P entries and gathers them
    (local pre-attention, no communication); the dense sub-sequence is the
    shards' sub-sequences in shard order -- (position, level) order again,
    since the shards are contiguous -- and it is attended causally on the slot
    index as one sequence (what ring attention computes); each shard's tokens
    take their outputs back from their own entries.  Returns the per-shard
    intermediates (lists) and the concatenated sub-sequence arrays."""
    sh = cp_shards(s, P)
    scale = default_scale(s, scale)
    q, k, v = (_f64(t).reshape(s.B, s.H, s.N, s.d) for t in (q, k, v))
    n = sh.N
    parts = []
    for r in range(P):
        qr, kr, vr = (t[:, :, r * n:(r + 1) * n] for t in (q, k, v))
        pq, pk, pv = (pyramid(sh, x) for x in (qr, kr, vr))
        sc = score(sh, qr, kr)
        idx, pos, slot = select(sh, sc)
        parts.append(dict(idx=idx, pos=pos + r * n, slot=slot,
                          qs=gather(sh, qr, pq, idx), ks=gather(sh, kr, pk, idx),
                          vs=gather(sh, vr, pv, idx)))
    cat = lambda key: np.concatenate([pt[key] for pt in parts], axis=2)
    qs, ks, vs = cat("qs"), cat("ks"), cat("vs")
    sfull = Shape(s.B, s.H, s.S, s.d, 2, 1, s.S)  # one sequence of S rows
    os_, lse = attn_fwd(sfull, qs, ks, vs, scale)
    o = np.concatenate([scatter(sh, os_[:, :, r * sh.S:(r + 1) * sh.S], parts[r]["slot"])
                        for r in range(P)], axis=2)
    return dict(parts=parts, qs=qs, ks=ks, vs=vs, os=os_, lse=lse, o=o, pos=cat("pos"),
                scale=scale, P=P, shard=sh)


def cp_backward(s: Shape, fwd: dict, dO) -> dict:
    """Backward of cp_forward: each shard's scatter-back adjoint, the attention
    backward over the concatenated sub-sequence, each shard's gather adjoint."""
    sh, P = fwd["shard"], fwd["P"]
    dO = _f64(dO).reshape(s.B, s.H, s.N, s.d)
    n = sh.N
    dos = np.concatenate([scatter_bwd(sh, dO[:, :, r * n:(r + 1) * n], fwd["parts"][r]["idx"],
                                      fwd["parts"][r]["slot"]) for r in range(P)], axis=2)
    sfull = Shape(s.B, s.H, s.S, s.d, 2, 1, s.S)
    dqs, dks, dvs = attn_bwd(sfull, fwd["qs"], fwd["ks"], fwd["vs"], dos, fwd["scale"])
    out = dict(dos=dos, dqs=dqs, dks=dks, dvs=dvs)
    for name, g in (("dq", dqs), ("dk", dks), ("dv", dvs)):
        out[name] = np.concatenate([gather_bwd(sh, g[:, :, r * sh.S:(r + 1) * sh.S],
                                               fwd["parts"][r]["slot"]) for r in range(P)], axis=2)
    return out
