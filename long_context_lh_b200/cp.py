"""Context-parallel Lighthouse: one GPU's shard of the layer and the ring.

[PT] bitsgeniais.com.br, "Adeus Custo Quadrático! ...", section "Escalando para
o Céu (ou 1 Milhão de Tokens!): Paralelismo de Contexto": for contexts beyond
one GPU the sequence is cut into P contiguous shards, one per GPU.  The
pyramid, the scores and the top-K selection run locally on each shard with no
communication; because the selected sub-sequence is dense, standard ring
attention runs on it.  This module drives one rank's part:

  * local pre-attention: the shard's pyramid + scores, its selection of S/P
    entries, the gather (the stage entry points of the C library, on the
    shard's N/P tokens);
  * ring attention over the global sub-sequence, the shards' sub-sequences in
    shard order (it is in (position, level) order again because the shards are
    contiguous): rank r's queries see every key block j < r in full and their
    own block causally.  The key/value blocks travel around the ring (P - 1
    steps, each a send to rank r+1 and a receive from rank r-1); each rank
    merges the block results into its running (output, log-sum-exp) in a fixed
    order, so the result is deterministic;
  * the backward: the same ring once more, each key block travelling with its
    dK, dV accumulators, which every rank that sees the block adds its
    contribution to; after P steps every block is home with its complete
    gradient.  dQ accumulates locally.  All sums run in a fixed order;
  * scatter-back and the gather adjoint, local.

The per-GPU arithmetic is in the C library (``CudaOps``: the stage calls and
lh_block_attn_fwd / _merge / _finish / _bwd, lh_accumulate); the transport is
``DistRing`` (torch.distributed point-to-point: NCCL between GPUs).  Nothing
here computes on the host.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import lighthouse as lh


# ------------------------------------------------------------------ transport
class DistRing:
    """Ring exchange over torch.distributed: each step sends this rank's tensors to
    rank r+1 and receives the same shapes from rank r-1 (all ranks take the same
    steps in the same order)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def exchange(self, tensors):
        if self.size == 1:
            return list(tensors)
        dist = self.dist
        nxt = (self.rank + 1) % self.size
        prv = (self.rank - 1) % self.size
        recv = [torch.empty_like(t) for t in tensors]
        ops = []
        for t, b in zip(tensors, recv):
            ops.append(dist.P2POp(dist.isend, t.contiguous(), self._peer(nxt), self.group))
            ops.append(dist.P2POp(dist.irecv, b, self._peer(prv), self.group))
        for w in dist.batch_isend_irecv(ops):
            w.wait()
        return recv

    def _peer(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)


# ------------------------------------------------------------ per-GPU pieces
@dataclass
class Front:
    """The shard's local pre-attention: selection and gathered rows."""
    idx: torch.Tensor
    pos: torch.Tensor
    slot: torch.Tensor
    qs: torch.Tensor
    ks: torch.Tensor
    vs: torch.Tensor
    inv_count: torch.Tensor | None = None


class CudaOps:
    """One GPU's steps, through the C library.  q, k, v of the shard: [B, H, N/P, d],
    bf16 or fp32, on the GPU; S_loc = S / P entries per shard."""

    def __init__(self, B, H, n_loc, d, p, L, s_loc, dtype: torch.dtype, scale: float = 0.0,
                 stream=None):
        self.shard = lh.make_shape(B, H, n_loc, d, p, L, s_loc)
        self.block = lh.make_shape(B, H, s_loc, d, 2, 1, s_loc)
        self.dt = lh.dtype_code(dtype)
        self.B, self.H, self.d, self.s_loc = B, H, d, s_loc
        self.rows = B * H * s_loc
        self.scale = scale
        self.stream = stream
        self.ws_bytes = lh.lh_attn_bwd_workspace_bytes(self.block)

    def _st(self):
        return self.stream if self.stream is not None else torch.cuda.current_stream().cuda_stream

    def front(self, q, k, v) -> Front:
        sh, dev = self.shard, q.device
        M = lh.lh_num_entries(sh)
        n_loc = sh.N
        npyr = max(self.B * self.H * (M - n_loc) * self.d, 1)
        pq, pk, pv = (torch.empty(npyr, dtype=torch.float32, device=dev) for _ in range(3))
        score = torch.empty(self.B * self.H * M, dtype=torch.float32, device=dev)
        idx = torch.empty((self.B, self.H, self.s_loc), dtype=torch.int32, device=dev)
        pos = torch.empty_like(idx)
        slot = torch.empty((self.B, self.H, M), dtype=torch.int32, device=dev)
        qs, ks, vs = (torch.empty((self.B, self.H, self.s_loc, self.d), dtype=torch.float16, device=dev)
                      for _ in range(3))
        st = self._st()
        lh.lh_build_pyramid_score(sh, self.dt, q, k, v, pq, pk, pv, score, st)
        lh.lh_topk_select(sh, score, idx, pos, slot, None, 0, st)
        lh.lh_gather(sh, self.dt, q, k, v, pq, pk, pv, idx, qs, ks, vs, st)
        return Front(idx, pos, slot, qs, ks, vs)

    def new_acc(self, qs):
        return (torch.empty((self.rows, self.d), dtype=torch.float32, device=qs.device),
                torch.empty(self.rows, dtype=torch.float32, device=qs.device))

    def attn_block(self, qs, ks, vs, causal: bool):
        os_ = torch.empty_like(qs)
        lse = torch.empty(self.rows, dtype=torch.float32, device=qs.device)
        lh.lh_block_attn_fwd(self.block, int(causal), qs, ks, vs, self.scale, os_, lse, self._st())
        return os_, lse

    def merge(self, acc, part, first: bool):
        lh.lh_block_attn_merge(self.rows, self.d, acc[0], acc[1], part[0], part[1], int(first),
                               self._st())

    def finish(self, acc, like):
        os_ = torch.empty_like(like)
        lh.lh_block_attn_finish(self.rows, self.d, acc[0], os_, self._st())
        return os_

    def scatter(self, fr: Front, os_, like):
        o = torch.empty_like(like)
        fr.inv_count = torch.empty((self.B, self.H, self.shard.N), dtype=torch.float32, device=o.device)
        lh.lh_scatter_back(self.shard, self.dt, os_, fr.slot, o, fr.inv_count, self._st())
        return o

    def scatter_bwd(self, fr: Front, dO):
        dos = torch.empty_like(fr.qs)
        lh.lh_scatter_back_bwd(self.shard, self.dt, dO, fr.slot, fr.inv_count, dos, self._st())
        return dos

    def zeros_grad(self, like):
        return torch.zeros(like.shape, dtype=torch.float32, device=like.device)

    def attn_block_bwd(self, qs, ks, vs, os_, lse, dos, causal: bool):
        dqs, dks, dvs = (torch.empty(qs.shape, dtype=torch.float32, device=qs.device) for _ in range(3))
        ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=qs.device)
        lh.lh_block_attn_bwd(self.block, int(causal), qs, ks, vs, os_, lse, dos, self.scale,
                             dqs, dks, dvs, ws, self.ws_bytes, self._st())
        return dqs, dks, dvs

    def accumulate(self, acc, x):
        lh.lh_accumulate(acc.numel(), acc, x, self._st())

    def gather_bwd(self, fr: Front, dqs, dks, dvs, like):
        dq, dk, dv = (torch.empty_like(like) for _ in range(3))
        lh.lh_gather_bwd(self.shard, self.dt, dqs, dks, dvs, fr.slot, dq, dk, dv, self._st())
        return dq, dk, dv


# ----------------------------------------------------------------- the ring
@dataclass
class CPSaved:
    front: Front
    os: torch.Tensor
    lse: torch.Tensor
    like: torch.Tensor  # an input of the shard (shape and dtype of the outputs)


def cp_forward(ops, ring, q, k, v):
    """This rank's shard of the layer's output, [B, H, N/P, d], and the state the
    backward needs.  Every rank calls it with its own shard, in rank order of
    the sequence (rank r holds tokens [r N/P, (r+1) N/P))."""
    r, P = ring.rank, ring.size
    fr = ops.front(q, k, v)
    acc = ops.new_acc(fr.qs)
    blk = [fr.ks, fr.vs]
    for step in range(P):
        j = (r - step) % P  # the rank whose key block this rank holds now
        if j <= r:  # key blocks after this rank's queries are never seen
            ops.merge(acc, ops.attn_block(fr.qs, blk[0], blk[1], causal=(j == r)), first=(step == 0))
        if step + 1 < P:
            blk = ring.exchange(blk)
    os_ = ops.finish(acc, fr.qs)
    o = ops.scatter(fr, os_, q)
    return o, CPSaved(fr, os_, acc[1], q)


def cp_backward(ops, ring, saved: CPSaved, dO):
    """dQ, dK, dV of this rank's shard.  Each key block goes once around the
    ring with its dK, dV accumulators: rank j's block collects the
    contributions of ranks j, j+1, ..., P-1 in that order and arrives back at
    rank j after P exchanges."""
    r, P = ring.rank, ring.size
    fr = saved.front
    dos = ops.scatter_bwd(fr, dO)
    dq_acc = ops.zeros_grad(fr.qs)
    blk = [fr.ks, fr.vs, ops.zeros_grad(fr.ks), ops.zeros_grad(fr.vs)]
    for step in range(P):
        j = (r - step) % P
        if j <= r:
            dqp, dkp, dvp = ops.attn_block_bwd(fr.qs, blk[0], blk[1], saved.os, saved.lse, dos,
                                               causal=(j == r))
            ops.accumulate(dq_acc, dqp)
            ops.accumulate(blk[2], dkp)
            ops.accumulate(blk[3], dvp)
        if step + 1 < P:
            blk = ring.exchange(blk)
        elif P > 1:  # the last hop only brings the gradients home
            blk = [None, None] + ring.exchange(blk[2:])
    return ops.gather_bwd(fr, dq_acc, blk[2], blk[3], saved.like)


def layer_forward(q, k, v, p: int, L: int, S: int, group=None, scale: float = 0.0):
    """The context-parallel layer on this rank's CUDA shard q, k, v [B, H, N/P, d]
    with a total budget of S entries (S/P per shard); returns (o, state)."""
    ring = DistRing(group)
    B, H, n_loc, d = q.shape
    if S % ring.size:
        raise ValueError("S must be a multiple of the number of ranks")
    ops = CudaOps(B, H, n_loc, d, p, L, S // ring.size, q.dtype, scale)
    o, saved = cp_forward(ops, ring, q, k, v)
    return o, (ops, ring, saved)


def layer_backward(state, dO):
    ops, ring, saved = state
    return cp_backward(ops, ring, saved, dO)
