"""The multi-GPU (N > 1) host path, on CPU with gloo ranks.

A multi-GPU run is N independent replicas of the workload (one batch per
rank, no collective on the data path); only the timing is combined, as the
max over ranks.  These tests run world-size-2 process groups on CPU: the
combination of timings, the per-rank batches, and what a rank that never
joins does to the others (an error within the group's timeout, not a hang).
"""
import multiprocessing as mp
import os
import socket
import traceback

import numpy as np
import pytest
import torch

import oracle
from long_context_lh_b200 import replicas
from long_context_lh_b200.synth import WORKLOADS, make_inputs

TINY = WORKLOADS["tiny"].with_(H=1, N=256, S=64, L=3)


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _env(rank, world, port):
    return {"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
            "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}


def _replica_output(rank):
    """What one rank computes: the layer's forward on its own batch (oracle, CPU)."""
    x = make_inputs(TINY, "cpu", with_dO=False, batch=rank)
    s = oracle.Shape(TINY.B, TINY.H, TINY.N, TINY.d, TINY.p, TINY.L, TINY.S)
    return oracle.forward(s, *(x[n].float().numpy() for n in ("q", "k", "v")))["o"]


def _worker(rank, world, port, out):
    try:
        os.environ.update(_env(rank, world, port))
        rk = replicas.from_env()
        replicas.init(rk, "gloo", timeout_s=60)
        try:
            step_ms = 1.5 * (rank + 1)  # this rank's (fake) device time
            job_ms = replicas.max_over_ranks(rk, step_ms)
            o = _replica_output(rank)
            replicas.barrier(rk)
            out.put((rank, job_ms, o))
        finally:
            replicas.finish(rk)
    except Exception:  # reported to the parent, which fails the test
        out.put((rank, "error", traceback.format_exc()))


def _run(world, target, *extra, timeout=120):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, out, *extra)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r = out.get(timeout=timeout)
            res[r[0]] = r[1:]
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return res


def test_two_ranks_combine_timing_and_keep_their_batches():
    res = _run(2, _worker)
    assert set(res) == {0, 1}
    for r in (0, 1):
        assert res[r][0] != "error", res[r][1]
        assert res[r][0] == pytest.approx(3.0)  # max over ranks, seen by every rank
    o0, o1 = res[0][1], res[1][1]
    assert not np.array_equal(o0, o1)  # independent batches
    for r in (0, 1):  # each replica equals the same computation in a single process
        np.testing.assert_array_equal(res[r][1], _replica_output(r))


def _lonely_worker(rank, world, port, out):
    """Rank 1 never joins; rank 0 must get an error, within its short timeout."""
    if rank == 1:
        out.put((1, "left", None))
        return
    try:
        os.environ.update(_env(rank, world, port))
        rk = replicas.from_env()
        replicas.init(rk, "gloo", timeout_s=5)
        try:
            replicas.max_over_ranks(rk, 1.0)
            out.put((0, "no error", None))
        finally:
            replicas.finish(rk)
    except Exception as e:  # the expected outcome
        out.put((0, "error", type(e).__name__))


def test_a_rank_that_never_joins_ends_the_others_with_an_error():
    res = _run(2, _lonely_worker, timeout=90)
    assert res[1][0] == "left"
    assert res[0][0] == "error", res[0]


def test_job_rate_and_rank_variables():
    assert replicas.job_rate(98304, 4, 0.5) == pytest.approx(4 * 98304 / 0.5)
    with pytest.raises(ValueError):
        replicas.job_rate(1, 1, 0.0)
    r = replicas.from_env({"RANK": "3", "WORLD_SIZE": "8", "LOCAL_RANK": "3"})
    assert (r.rank, r.world, r.local_rank, r.multi) == (3, 8, 3, True)
    assert not replicas.from_env({}).multi
    with pytest.raises(ValueError):
        replicas.from_env({"RANK": "2", "WORLD_SIZE": "2"})
    assert replicas.max_over_ranks(replicas.from_env({}), 2.5) == 2.5  # one process: identity


def test_batch_zero_is_the_default_draw():
    a = make_inputs(TINY, "cpu", with_dO=False)
    b = make_inputs(TINY, "cpu", with_dO=False, batch=0)
    c = make_inputs(TINY, "cpu", with_dO=False, batch=1)
    assert torch.equal(a["q"], b["q"]) and not torch.equal(a["q"], c["q"])
