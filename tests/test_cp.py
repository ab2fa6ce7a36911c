"""Context-parallel Lighthouse (long_context_lh_b200/cp.py): the ring.

CPU (gloo, world sizes 2 and 4): every rank runs cp_forward / cp_backward on
its shard with the ring exchanging real tensors through torch.distributed; the
per-GPU block steps are stood in for by a small fp64 numpy implementation
defined here (textbook softmax attention of one block pair, the log-sum-exp
merge, the fixed-order sums) and by the oracle's shard-local stages.  The
concatenated outputs and gradients must equal the oracle's context-parallel
layer (oracle.cp_forward / cp_backward: per-shard selection, one causal
attention over the concatenated sub-sequence) to fp64 rounding -- which checks
the ring's schedule (who sees which key block, in which order), the merge and
the travelling gradient accumulators.

GPU (one device): the same ring with the CUDA library's block calls, P ranks
run as threads of one process exchanging through a local ring (the ranks never
wait on one another inside a kernel), against the same oracle at the attention
tolerance.
"""
import os
import socket
import threading

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from long_context_lh_b200 import cp
from long_context_lh_b200.synth import WORKLOADS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ------------------------------------------------ fp64 stand-in for the GPU steps
class NumpyOps:
    """The per-GPU steps in fp64 on the CPU (test stand-in for cp.CudaOps)."""

    def __init__(self, shard: oracle.Shape, scale: float):
        self.sh, self.scale = shard, scale

    def front(self, q, k, v):
        sh = self.sh
        qn, kn, vn = (t.double().numpy() for t in (q, k, v))
        pq, pk, pv = (oracle.pyramid(sh, x) for x in (qn, kn, vn))
        idx, pos, slot = oracle.select(sh, oracle.score(sh, qn, kn))
        g = lambda x, pyr: torch.from_numpy(oracle.gather(sh, x, pyr, idx))
        return cp.Front(torch.from_numpy(idx), torch.from_numpy(pos), torch.from_numpy(slot),
                        g(qn, pq), g(kn, pk), g(vn, pv))

    def new_acc(self, qs):
        B, H, S, d = qs.shape
        return torch.zeros((B * H * S, d), dtype=torch.float64), torch.zeros(B * H * S, dtype=torch.float64)

    def _logits(self, qs, ks, causal):
        z = self.scale * np.einsum("bhqd,bhkd->bhqk", qs.numpy(), ks.numpy())
        if causal:
            S = z.shape[-1]
            z = np.where(np.arange(S)[None, :] <= np.arange(S)[:, None], z, -np.inf)
        return z

    def attn_block(self, qs, ks, vs, causal):
        z = self._logits(qs, ks, causal)
        m = z.max(-1, keepdims=True)
        e = np.exp(z - m)
        s = e.sum(-1, keepdims=True)
        o = np.einsum("bhqk,bhkd->bhqd", e / s, vs.numpy())
        return torch.from_numpy(o), torch.from_numpy((m + np.log(s))[..., 0].reshape(-1))

    def merge(self, acc, part, first):
        o, lse = part
        o = o.reshape(acc[0].shape)
        if first:
            acc[0].copy_(o)
            acc[1].copy_(lse)
            return
        m = torch.maximum(acc[1], lse)
        wa, wb = torch.exp(acc[1] - m), torch.exp(lse - m)
        acc[0].copy_((acc[0] * wa[:, None] + o * wb[:, None]) / (wa + wb)[:, None])
        acc[1].copy_(m + torch.log(wa + wb))

    def finish(self, acc, like):
        return acc[0].reshape(like.shape).clone()

    def scatter(self, fr, os_, like):
        return torch.from_numpy(oracle.scatter(self.sh, os_.numpy(), fr.slot.numpy()))

    def scatter_bwd(self, fr, dO):
        return torch.from_numpy(oracle.scatter_bwd(self.sh, dO.double().numpy(), fr.idx.numpy(),
                                                   fr.slot.numpy()))

    def zeros_grad(self, like):
        return torch.zeros(like.shape, dtype=torch.float64)

    def attn_block_bwd(self, qs, ks, vs, os_, lse, dos, causal):
        z = self._logits(qs, ks, causal)
        p = np.exp(z - lse.numpy().reshape(z.shape[:-1])[..., None])
        do, o = dos.numpy(), os_.numpy()
        dp = np.einsum("bhqd,bhkd->bhqk", do, vs.numpy())
        dsum = np.einsum("bhqd,bhqd->bhq", do, o)
        ds = p * (dp - dsum[..., None])
        dq = self.scale * np.einsum("bhqk,bhkd->bhqd", ds, ks.numpy())
        dk = self.scale * np.einsum("bhqk,bhqd->bhkd", ds, qs.numpy())
        dv = np.einsum("bhqk,bhqd->bhkd", p, do)
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)

    def accumulate(self, acc, x):
        acc += x

    def gather_bwd(self, fr, dqs, dks, dvs, like):
        return tuple(torch.from_numpy(oracle.gather_bwd(self.sh, g.numpy(), fr.slot.numpy()))
                     for g in (dqs, dks, dvs))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, shape, seed, outdir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        s = oracle.Shape(*shape)
        rng = np.random.default_rng(seed)
        q, k, v, dO = (rng.standard_normal((s.B, s.H, s.N, s.d)) for _ in range(4))
        n = s.N // world
        mine = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, rank * n:(rank + 1) * n]))
        ring = cp.DistRing()
        ops = NumpyOps(oracle.cp_shards(s, world), oracle.default_scale(s))
        o, saved = cp.cp_forward(ops, ring, mine(q), mine(k), mine(v))
        dq, dk, dv = cp.cp_backward(ops, ring, saved, mine(dO))
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), o=o.numpy(), dq=dq.numpy(),
                 dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ring_on_gloo_equals_the_oracle_layer(world, tmp_path):
    shape = (1, 2, 1024, 8, 2, 3, 192)  # B, H, N, d, p, L, S: shards of 1024/P tokens, S/P entries
    seed = 11 + world
    mp.start_processes(_rank_main, args=(world, _free_port(), shape, seed, str(tmp_path)),
                       nprocs=world, start_method="spawn")
    s = oracle.Shape(*shape)
    rng = np.random.default_rng(seed)
    q, k, v, dO = (rng.standard_normal((s.B, s.H, s.N, s.d)) for _ in range(4))
    ref = oracle.cp_forward(s, q, k, v, world)
    bref = oracle.cp_backward(s, ref, dO)
    got = [np.load(os.path.join(tmp_path, f"rank{r}.npz")) for r in range(world)]
    for name, want in (("o", ref["o"]), ("dq", bref["dq"]), ("dk", bref["dk"]), ("dv", bref["dv"])):
        cat = np.concatenate([g[name] for g in got], axis=2)
        assert np.abs(cat - want).max() <= 1e-10 * (1 + np.abs(want).max()), name


# ------------------------------------------------------------------- one GPU
class LocalRing:
    """P ranks as threads of one process: exchange() hands each rank's tensors to
    the next rank (host-side barrier; no kernel waits on another rank)."""

    def __init__(self, P):
        self.P, self.slots, self.bar = P, [None] * P, threading.Barrier(P)

    def rank_view(self, r):
        ring = self

        class View:
            rank, size = r, ring.P

            def exchange(self, tensors):
                ring.bar.wait()
                ring.slots[(r + 1) % ring.P] = list(tensors)
                ring.bar.wait()
                out = ring.slots[r]
                ring.bar.wait()
                return out
        return View()


@pytest.mark.gpu
@pytest.mark.parametrize("P,case", [(2, dict(dtype="bf16", dist="outliers", N=8192, S=1024, L=4, H=2)),
                                    (4, dict(dtype="bf16", N=8192, S=1024, L=3, H=2)),
                                    (4, dict(dtype="bf16", d=128, p=2, L=4, N=4096, S=640, H=1)),
                                    (2, dict(dtype="bf16", N=4096, S=200, L=3, H=1))],
                         ids=["p2", "p4", "p4-d128", "p2-ragged"])
def test_ring_on_one_gpu_matches_the_oracle(P, case):
    from long_context_lh_b200 import lighthouse as lh
    w = WORKLOADS["tiny"].with_(**case)
    xc = make_inputs(w, "cpu")
    dev = torch.device("cuda:0")
    n = w.N // P
    ring = LocalRing(P)
    results, errors = [None] * P, []

    def rank(r):
        try:
            torch.cuda.set_device(dev)
            sl = lambda t: t[:, :, r * n:(r + 1) * n].contiguous().to(dev)
            q, k, v, dO = (sl(xc[x]) for x in ("q", "k", "v", "dO"))
            ops = cp.CudaOps(w.B, w.H, n, w.d, w.p, w.L, w.S // P, q.dtype)
            view = ring.rank_view(r)
            o, saved = cp.cp_forward(ops, view, q, k, v)
            grads = cp.cp_backward(ops, view, saved, dO)
            torch.cuda.synchronize()
            results[r] = [t.double().cpu() for t in (o,) + tuple(grads)]
        except Exception as e:  # noqa: BLE001 -- reported below
            errors.append(e)
            ring.bar.abort()

    threads = [threading.Thread(target=rank, args=(r,)) for r in range(P)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert lh.lh_read_device_status() == 0
    s = oracle.Shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)
    f = [xc[x].float().numpy() for x in ("q", "k", "v", "dO")]
    ref = oracle.cp_forward(s, *f[:3], P)
    bref = oracle.cp_backward(s, ref, f[3])
    for i, (name, want) in enumerate((("o", ref["o"]), ("dq", bref["dq"]), ("dk", bref["dk"]),
                                      ("dv", bref["dv"]))):
        got = torch.cat([res[i] for res in results], dim=2).numpy()
        err = np.abs(got - want)
        # the layer's results are stored in bf16: 2e-2 plus half a bf16 ulp
        assert np.all(err <= 2e-2 + 2.0 ** -8 * np.abs(want)), f"{name}: max err {err.max():.4g}"
        assert err.mean() <= 1e-2 * np.abs(want).mean(), f"{name}: mean relative error"
