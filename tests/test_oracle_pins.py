"""Pins for the CPU oracle against things other than itself.

Each test ties one oracle stage to a closed form, a brute force, a library
routine (torch SDPA in fp64), finite differences, an adjoint identity or the
hand-worked fixture in tests/golden/, so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails here.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import Shape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def rand_qkv(s: Shape, scale=1.0, bf16=True):
    out = []
    for _ in range(3):
        x = rng.standard_normal((s.B, s.H, s.N, s.d)).astype(np.float32) * scale
        out.append(bf16_round(x) if bf16 else x)
    return out


# ------------------------------------------------------------------ pyramid
@pytest.mark.parametrize("p,L", [(2, 4), (4, 3), (3, 3), (8, 2)])
def test_pyramid_equals_direct_span_mean(p, L):
    """Hierarchical average == plain mean over the p^l tokens of the span."""
    N = p ** (L - 1) * 5
    s = Shape(2, 2, N, 16, p, L, 4)
    x = rng.standard_normal((s.B, s.H, N, s.d))
    pyr = oracle.pyramid(s, x)
    for l in range(1, L):
        w = p ** l
        direct = x.reshape(s.B, s.H, N // w, w, s.d).mean(axis=3)
        got = pyr[:, :, s.level_off(l) - N: s.level_off(l) - N + N // w]
        np.testing.assert_allclose(got, direct, rtol=1e-12, atol=1e-13)


def test_pyramid_constant_and_linear():
    s = Shape(1, 3, 64, 8, 4, 4, 4)
    c = np.full((1, 3, 64, 8), 0.375)
    assert np.all(oracle.pyramid(s, c) == 0.375)
    a, b = rng.standard_normal((2, 1, 3, 64, 8))
    lhs = oracle.pyramid(s, 2.5 * a - 1.25 * b)
    rhs = 2.5 * oracle.pyramid(s, a) - 1.25 * oracle.pyramid(s, b)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


# -------------------------------------------------------------------- score
@pytest.mark.parametrize("d,bf16", [(64, True), (128, True), (64, False), (8, True)])
def test_score_close_to_fp64_norms(d, bf16):
    """fp32 canonical-order norms agree with exact fp64 norms to a few ulp."""
    s = Shape(1, 2, 256, d, 4, 3, 16)
    q, k, _ = rand_qkv(s, 3.0, bf16)
    sc = oracle.score(s, q, k)
    exact = (np.linalg.norm(q.astype(np.float64), axis=-1)
             + np.linalg.norm(k.astype(np.float64), axis=-1))
    rel = np.abs(sc[:, :, :s.N] - exact) / exact
    # d/8 + log2(d/8) fp32 roundings in the sum of squares, 2 in the roots, 1 in the sum
    assert rel.max() < (d + 8) * 2.0 ** -24


def test_score_maxpool_inheritance_exact():
    """score at level l equals the max of level-0 scores over the span, bit for bit."""
    s = Shape(2, 2, 512, 64, 2, 5, 16)
    q, k, _ = rand_qkv(s)
    sc = oracle.score(s, q, k)
    lvl0 = sc[:, :, :s.N]
    for l in range(1, s.L):
        w = s.p ** l
        want = lvl0.reshape(s.B, s.H, s.N // w, w).max(axis=-1)
        got = sc[:, :, s.level_off(l): s.level_off(l) + s.N // w]
        assert np.array_equal(got, want)


def test_score_uses_both_q_and_k():
    """Zeroing K leaves ||Q||; zeroing Q leaves ||K|| (catches a dropped term)."""
    s = Shape(1, 1, 64, 64, 4, 2, 8)
    q, k, _ = rand_qkv(s)
    z = np.zeros_like(q)
    sq = oracle.score(s, q, z)[..., :s.N]
    sk = oracle.score(s, z, k)[..., :s.N]
    np.testing.assert_allclose(sq, np.linalg.norm(q, axis=-1), rtol=1e-6)
    np.testing.assert_allclose(sk, np.linalg.norm(k, axis=-1), rtol=1e-6)


# ---------------------------------------------------------------- selection
def brute_select(s: Shape, sc_unit: np.ndarray):
    """Pure-Python reference: sort all entries by (score desc, gid asc)."""
    M = s.M
    ranked = sorted(range(M), key=lambda g: (-float(sc_unit[g]), g))[: s.S]
    items = []
    for g in ranked:
        l = max(l for l in range(s.L) if g >= s.level_off(l))
        j = g - s.level_off(l)
        items.append(((j + 1) * s.p ** l - 1, l, g))
    items.sort()
    return [g for _, _, g in items], [pp for pp, _, _ in items]


@pytest.mark.parametrize("p,L,S", [(2, 3, 7), (4, 3, 40), (3, 2, 11), (2, 1, 9)])
def test_select_brute_force(p, L, S):
    N = p ** (L - 1) * 12
    s = Shape(1, 2, N, 8, p, L, S)
    q, k, _ = rand_qkv(s)
    # quantise to create many exact score ties, beyond the inherited ones
    q = np.round(q * 2) / 2
    k = np.round(k * 2) / 2
    sc = oracle.score(s, q, k)
    idx, pos, slot = oracle.select(s, sc)
    for h in range(s.H):
        gids, poss = brute_select(s, sc[0, h])
        assert idx[0, h].tolist() == gids
        assert pos[0, h].tolist() == poss


def test_select_invariants():
    s = Shape(1, 3, 1024, 64, 4, 4, 100)
    q, k, _ = rand_qkv(s)
    sc = oracle.score(s, q, k)
    idx, pos, slot = oracle.select(s, sc)
    for h in range(s.H):
        g = idx[0, h]
        assert len(set(g.tolist())) == s.S
        keys = [(float(sc[0, h, x]), -int(x)) for x in range(s.M)]
        sel = set(g.tolist())
        assert min(keys[x] for x in sel) > max(keys[x] for x in range(s.M) if x not in sel)
        # (pos, level) strictly increasing, pos non-decreasing
        lv = np.array([max(l for l in range(s.L) if x >= s.level_off(l)) for x in g])
        pp = pos[0, h]
        assert np.all(np.diff(pp) >= 0)
        assert all((pp[i], lv[i]) < (pp[i + 1], lv[i + 1]) for i in range(s.S - 1))
        # slot is the inverse map
        sl = slot[0, h]
        assert np.all(sl[g] == np.arange(s.S))
        assert np.sum(sl >= 0) == s.S
        # closure: a selected coarse entry's argmax child (lowest index) is selected
        for x in g:
            l = max(l for l in range(s.L) if x >= s.level_off(l))
            if l == 0:
                continue
            j = x - s.level_off(l)
            ch = s.level_off(l - 1) + s.p * j + np.arange(s.p)
            best = ch[np.argmax(sc[0, h, ch])]  # argmax returns the first maximum
            assert best in sel


def test_select_L1_is_topS_tokens_in_order():
    s = Shape(1, 1, 200, 16, 2, 1, 50)
    q, k, _ = rand_qkv(s)
    sc = oracle.score(s, q, k)
    idx, pos, _ = oracle.select(s, sc)
    want = np.sort(np.argsort(-sc[0, 0], kind="stable")[:50])
    assert np.array_equal(idx[0, 0], want)
    assert np.array_equal(pos[0, 0], want)


def test_worked_example_fixture():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    s = Shape(**g["shape"])
    q = np.zeros((1, 1, s.N, s.d), np.float32)
    k = np.zeros_like(q)
    q[0, 0, :, 0] = g["q_scale_axis0"]
    k[0, 0, :, 1] = g["k_scale_axis1"]
    sc = oracle.score(s, q, k)
    assert sc[0, 0].tolist() == g["score"]
    idx, pos, slot = oracle.select(s, sc)
    assert idx[0, 0].tolist() == g["idx"]
    assert pos[0, 0].tolist() == g["pos"]
    ramp = np.repeat(np.arange(1, s.S + 1, dtype=np.float64)[:, None], s.d, 1)[None, None]
    o = oracle.scatter(s, ramp, slot)
    assert np.allclose(o[0, 0, :, 0], g["scatter_of_ramp"])
    ones = np.ones((1, 1, s.N, s.d))
    # contributor counts: scatter_bwd of ones sums 1/c_t over each span
    dos = oracle.scatter_bwd(s, ones, idx, slot)
    c = np.array(g["contributors"], np.float64)
    for kk, gid in enumerate(g["idx"]):
        l = max(l for l in range(s.L) if gid >= s.level_off(l))
        j = gid - s.level_off(l)
        span = range(j * s.p ** l, (j + 1) * s.p ** l)
        assert math.isclose(dos[0, 0, kk, 0], sum(1.0 / c[t] for t in span))


# ------------------------------------------------------------------- gather
def test_gather_rows_are_pyramid_rows():
    s = Shape(1, 2, 256, 8, 4, 3, 30)
    q, k, v = rand_qkv(s)
    sc = oracle.score(s, q, k)
    idx, _, _ = oracle.select(s, sc)
    pv = oracle.pyramid(s, v)
    vs = oracle.gather(s, v, pv, idx)
    full = np.concatenate([v.astype(np.float64), pv], axis=2)
    for h in range(s.H):
        assert np.array_equal(vs[0, h], full[0, h, idx[0, h]])


# ---------------------------------------------------------------- attention
def sdpa64(qs, ks, vs, scale):
    t = [torch.from_numpy(np.asarray(x, np.float64)) for x in (qs, ks, vs)]
    return torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True, scale=scale)


def test_attention_fwd_matches_torch_sdpa():
    s = Shape(2, 2, 96, 16, 2, 2, 80)
    qs, ks, vs = (rng.standard_normal((2, 2, 80, 16)) * 1.5 for _ in range(3))
    sc = 0.3
    os_, lse = oracle.attn_fwd(s, qs, ks, vs, sc)
    ref = sdpa64(qs, ks, vs, sc).numpy()
    np.testing.assert_allclose(os_, ref, rtol=1e-11, atol=1e-12)
    z = sc * np.einsum("bhid,bhjd->bhij", qs, ks)
    z = np.where(np.tril(np.ones((80, 80), bool)), z, -np.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(z), -1).numpy(), rtol=1e-12)
    rows = np.array([0, 5, 79], np.int32)
    os_r, lse_r = oracle.attn_fwd(s, qs, ks, vs, sc, rows=rows)
    np.testing.assert_array_equal(os_r, os_[:, :, rows])


def test_attention_bwd_matches_torch_autograd():
    s = Shape(1, 2, 64, 16, 2, 2, 48)
    qs, ks, vs, dos = (rng.standard_normal((1, 2, 48, 16)) for _ in range(4))
    sc = 0.25
    dq, dk, dv = oracle.attn_bwd(s, qs, ks, vs, dos, sc)
    t = [torch.from_numpy(x).requires_grad_(True) for x in (qs, ks, vs)]
    out = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True, scale=sc)
    out.backward(torch.from_numpy(dos))
    for got, ref in zip((dq, dk, dv), t):
        np.testing.assert_allclose(got, ref.grad.numpy(), rtol=1e-10, atol=1e-11)


# ------------------------------------------------------------ scatter-back
def test_scatter_L1_is_permutation():
    s = Shape(1, 1, 40, 4, 2, 1, 13)
    q, k, _ = rand_qkv(s)
    idx, _, slot = oracle.select(s, oracle.score(s, q, k))
    os_ = rng.standard_normal((1, 1, 13, 4))
    o = oracle.scatter(s, os_, slot)
    for t in range(40):
        sl = slot[0, 0, t]
        want = os_[0, 0, sl] if sl >= 0 else np.zeros(4)
        assert np.array_equal(o[0, 0, t], want)


def test_scatter_constant_rows():
    s = Shape(1, 2, 256, 8, 4, 4, 37)
    q, k, _ = rand_qkv(s)
    idx, _, slot = oracle.select(s, oracle.score(s, q, k))
    o = oracle.scatter(s, np.full((1, 2, 37, 8), 0.625), slot)
    covered = np.zeros((1, 2, 256), bool)
    for h in range(2):
        for t in range(256):
            covered[0, h, t] = any(slot[0, h, s.level_off(l) + t // s.p ** l] >= 0
                                   for l in range(s.L))
    assert np.all(o[covered] == 0.625)
    assert np.all(o[~covered] == 0.0)


@pytest.mark.parametrize("p,L,S", [(2, 3, 9), (4, 3, 21)])
def test_adjoint_identities(p, L, S):
    """<scatter(Y), Z> = <Y, scatter_bwd(Z)> and <gather(pyramid X), W> = <X, gather_bwd(W)>."""
    N = p ** (L - 1) * 6
    s = Shape(1, 2, N, 8, p, L, S)
    q, k, _ = rand_qkv(s)
    idx, _, slot = oracle.select(s, oracle.score(s, q, k))
    Y = rng.standard_normal((1, 2, S, 8))
    Z = rng.standard_normal((1, 2, N, 8))
    lhs = np.sum(oracle.scatter(s, Y, slot) * Z)
    rhs = np.sum(Y * oracle.scatter_bwd(s, Z, idx, slot))
    assert math.isclose(lhs, rhs, rel_tol=1e-12)
    X = rng.standard_normal((1, 2, N, 8))
    W = rng.standard_normal((1, 2, S, 8))
    lhs = np.sum(oracle.gather(s, X, oracle.pyramid(s, X), idx) * W)
    rhs = np.sum(X * oracle.gather_bwd(s, W, slot))
    assert math.isclose(lhs, rhs, rel_tol=1e-12)


# ------------------------------------------------------- whole-pipeline pins
def test_pipeline_finite_differences():
    """Backward of the whole layer (selection frozen) vs fp64 central differences."""
    s = Shape(1, 1, 16, 4, 2, 3, 9)
    q, k, v = rand_qkv(s)
    fwd = oracle.forward(s, q, k, v)
    G = rng.standard_normal((1, 1, s.N, s.d))
    bwd = oracle.backward(s, fwd, G)
    base = [x.astype(np.float64) for x in (q, k, v)]
    eps = 1e-6
    for which, name in enumerate(("dq", "dk", "dv")):
        num = np.zeros_like(base[which])
        for t in range(s.N):
            for c in range(s.d):
                vals = []
                for sgn in (1, -1):
                    xs = [b.copy() for b in base]
                    xs[which][0, 0, t, c] += sgn * eps
                    o = oracle.forward_fixed(s, *xs, fwd["idx"], fwd["slot"], fwd["scale"])
                    vals.append(np.sum(o * G))
                num[0, 0, t, c] = (vals[0] - vals[1]) / (2 * eps)
        np.testing.assert_allclose(bwd[name], num, rtol=1e-6, atol=1e-8)


def test_degenerate_L1_full_selection_is_causal_sdpa():
    """L = 1 and S = N: every token selected in order, so the layer is causal SDPA."""
    s = Shape(1, 2, 64, 16, 2, 1, 64)
    q, k, v = rand_qkv(s)
    fwd = oracle.forward(s, q, k, v)
    assert np.array_equal(fwd["idx"][0, 0], np.arange(64))
    t = [torch.from_numpy(x.astype(np.float64)).requires_grad_(True) for x in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True)
    np.testing.assert_allclose(fwd["o"], ref.detach().numpy(), rtol=1e-11, atol=1e-12)
    G = rng.standard_normal((1, 2, 64, 16))
    ref.backward(torch.from_numpy(G))
    bwd = oracle.backward(s, fwd, G)
    for name, r in zip(("dq", "dk", "dv"), t):
        np.testing.assert_allclose(bwd[name], r.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_no_gradient_through_selection():
    """Perturbing scores without changing the selected set leaves outputs unchanged."""
    s = Shape(1, 1, 64, 8, 2, 3, 12)
    q, k, v = rand_qkv(s)
    fwd = oracle.forward(s, q, k, v)
    o_fixed = oracle.forward_fixed(s, q, k, v, fwd["idx"], fwd["slot"], fwd["scale"])
    assert np.array_equal(o_fixed, fwd["o"])


@pytest.mark.parametrize("S,chunk", [(96, 32), (130, 1024)])
def test_attention_bwd_sampled_matches_full_backward_and_autograd(S, chunk):
    """The sampled-row/column backward equals the oracle's full backward (C loops)
    and torch autograd in fp64 at every sampled position, including the first
    and last rows and a block boundary."""
    rng = np.random.default_rng(11)
    d = 16
    q, k, v, do = (rng.standard_normal((S, d)) for _ in range(4))
    sc = 1.0 / np.sqrt(d)
    rows = np.array([0, 1, 31, 32, 33, S // 2, S - 2, S - 1])
    dq, dk, dv = oracle.attn_bwd_sampled(q, k, v, do, sc, rows, chunk=chunk)
    s = oracle.Shape(1, 1, S, d, 2, 1, S)
    fq, fk, fv = (x[0, 0] for x in oracle.attn_bwd(s, q[None, None], k[None, None],
                                                   v[None, None], do[None, None], sc))
    for got, full in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(got, full[rows], rtol=1e-10, atol=1e-12)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=sc)
    out.backward(torch.tensor(do))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.numpy()[rows], rtol=1e-10, atol=1e-12)


# --------------------------------------------------- variants (ablations, keep-coarsest)
@pytest.mark.parametrize("d", [64, 128, 8])
def test_score_modes_close_to_fp64_closed_forms(d):
    """The product of the two norms and the norm of [q; k] agree with exact fp64
    values to a few ulp, and coarse levels still inherit the exact span max."""
    s = Shape(1, 2, 256, d, 4, 3, 16)
    q, k, _ = rand_qkv(s, 3.0, True)
    nq = np.linalg.norm(q.astype(np.float64), axis=-1)
    nk = np.linalg.norm(k.astype(np.float64), axis=-1)
    for mode, exact in ((oracle.SCORE_PRODUCT, nq * nk), (oracle.SCORE_CONCAT, np.sqrt(nq ** 2 + nk ** 2))):
        sc = oracle.score(s, q, k, mode=mode)
        rel = np.abs(sc[:, :, :s.N] - exact) / exact
        assert rel.max() < (d + 8) * 2.0 ** -24, mode
        lvl0 = sc[:, :, :s.N]
        for l in range(1, s.L):
            w = s.p ** l
            got = sc[:, :, s.level_off(l): s.level_off(l) + s.N // w]
            assert np.array_equal(got, lvl0.reshape(s.B, s.H, s.N // w, w).max(axis=-1))


def test_score_modes_special_cases():
    """Zero K: the product is 0 and the concatenation's norm is ||q|| (as the sum's);
    q = k: the product is ||q||^2 and the concatenation sqrt(2) ||q||."""
    s = Shape(1, 1, 64, 64, 4, 2, 8)
    q, _, _ = rand_qkv(s)
    z = np.zeros_like(q)
    n = np.linalg.norm(q.astype(np.float64), axis=-1)
    assert np.all(oracle.score(s, q, z, mode=oracle.SCORE_PRODUCT)[..., :s.N] == 0)
    np.testing.assert_allclose(oracle.score(s, q, z, mode=oracle.SCORE_CONCAT)[..., :s.N], n, rtol=1e-6)
    np.testing.assert_allclose(oracle.score(s, q, q, mode=oracle.SCORE_PRODUCT)[..., :s.N], n ** 2, rtol=1e-5)
    np.testing.assert_allclose(oracle.score(s, q, q, mode=oracle.SCORE_CONCAT)[..., :s.N], np.sqrt(2) * n, rtol=1e-6)


@pytest.mark.parametrize("p,L,S", [(2, 3, 40), (4, 3, 30), (3, 2, 20), (4, 2, 12)])
def test_select_keep_coarsest_brute_force(p, L, S):
    """Keep-coarsest: every level-(L-1) entry is selected; the remaining
    S - n_{L-1} slots hold the largest (score, -gid) keys of the other levels
    (pure-Python sort); the order is (pos, level) as usual."""
    N = p ** (L - 1) * 12
    s = Shape(1, 2, N, 8, p, L, S)
    q, k, _ = rand_qkv(s)
    sc = oracle.score(s, q, k)
    idx, pos, slot = oracle.select(s, sc, keep_coarsest=True)
    top = s.level_off(L - 1)
    ncoarse = s.M - top
    assert ncoarse <= S
    for h in range(s.H):
        g = idx[0, h].tolist()
        assert set(range(top, s.M)) <= set(g)
        rest = sorted(range(top), key=lambda e: (-float(sc[0, h, e]), e))[: S - ncoarse]
        assert set(g) == set(rest) | set(range(top, s.M))
        items = []
        for e in g:
            l = max(l for l in range(s.L) if e >= s.level_off(l))
            items.append(((e - s.level_off(l) + 1) * s.p ** l - 1, l))
        assert items == sorted(items) and pos[0, h].tolist() == [it[0] for it in items]
        for kk, e in enumerate(g):
            assert slot[0, h, e] == kk
    # every token then has a contributor: the scatter-back count is >= 1 everywhere
    o = oracle.scatter(s, np.ones((1, 2, S, 8)), slot)
    assert np.all(o == 1.0)


def entry_centric_scatter(s: Shape, os_unit, idx_unit, mode):
    """Scatter-back written from the entries' side: entry e (slot k) reaches every
    token of its span (mean, sum) or only pos(e) (last); row t of the N x S
    weight matrix is then normalised by its count (mean, last) or not (sum)."""
    W = np.zeros((s.N, s.S))
    for kk, g in enumerate(idx_unit):
        l = max(l for l in range(s.L) if g >= s.level_off(l))
        j = g - s.level_off(l)
        w = s.p ** l
        toks = [(j + 1) * w - 1] if mode == oracle.SCATTER_LAST else range(j * w, (j + 1) * w)
        for t in toks:
            W[t, kk] = 1.0
    if mode != oracle.SCATTER_SUM:
        c = W.sum(axis=1, keepdims=True)
        W = np.divide(W, c, out=np.zeros_like(W), where=c > 0)
    return W @ os_unit


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("p,L,S", [(2, 4, 30), (4, 3, 40), (3, 3, 25)])
def test_scatter_modes_entry_centric_and_adjoint(mode, p, L, S):
    """Each scatter mode equals the entry-side construction above, and its
    backward is its exact adjoint: <scatter(Y), Z> = <Y, scatter_bwd(Z)>."""
    N = p ** (L - 1) * 6
    s = Shape(1, 2, N, 8, p, L, S)
    q, k, _ = rand_qkv(s)
    idx, _, slot = oracle.select(s, oracle.score(s, q, k))
    Y = rng.standard_normal((1, 2, S, 8))
    Z = rng.standard_normal((1, 2, N, 8))
    o = oracle.scatter(s, Y, slot, mode)
    for h in range(2):
        np.testing.assert_allclose(o[0, h], entry_centric_scatter(s, Y[0, h], idx[0, h], mode),
                                   rtol=1e-12, atol=1e-12)
    lhs = np.sum(o * Z)
    rhs = np.sum(Y * oracle.scatter_bwd(s, Z, idx, slot, mode))
    assert math.isclose(lhs, rhs, rel_tol=1e-12)
    if mode == oracle.SCATTER_LAST:  # causal: a token receives nothing from entries ending later
        for h in range(2):
            for t in range(N):
                for l in range(L):
                    e = slot[0, h, s.level_off(l) + t // p ** l]
                    if e >= 0 and (t + 1) % p ** l:
                        Yp = Y.copy()
                        Yp[0, h, e] += 1.0
                        assert np.array_equal(oracle.scatter(s, Yp, slot, mode)[0, h, t], o[0, h, t])
                        break
                else:
                    continue
                break


# ------------------------------------------------------- context parallelism
def test_cp_one_shard_is_the_layer():
    """One shard: the context-parallel layer is the single-GPU layer, bit for bit."""
    s = Shape(1, 2, 512, 8, 4, 3, 96)
    rng = np.random.default_rng(21)
    q, k, v, dO = (rng.standard_normal((1, 2, 512, 8)) for _ in range(4))
    a, b = oracle.forward(s, q, k, v), oracle.cp_forward(s, q, k, v, 1)
    assert np.array_equal(a["o"], b["o"])
    ga, gb = oracle.backward(s, a, dO), oracle.cp_backward(s, b, dO)
    for n in ("dq", "dk", "dv"):
        assert np.array_equal(ga[n], gb[n])


@pytest.mark.parametrize("P", [2, 4])
def test_cp_full_selection_is_causal_sdpa_over_the_whole_sequence(P):
    """L = 1 and S = N: every shard selects all of its tokens, the concatenated
    sub-sequence is the whole sequence in order, and the layer is causal SDPA over
    all N tokens (forward and gradients, torch fp64 autograd) whatever the shard
    count -- the shards only split the work."""
    N, d = 256, 8
    s = Shape(1, 2, N, d, 2, 1, N)
    rng = np.random.default_rng(5 + P)
    q, k, v, dO = (rng.standard_normal((1, 2, N, d)) for _ in range(4))
    f = oracle.cp_forward(s, q, k, v, P)
    g = oracle.cp_backward(s, f, dO)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    ref.backward(torch.tensor(dO))
    assert np.allclose(f["o"], ref.detach().numpy(), atol=1e-12)
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        assert np.allclose(g[name], t.grad.numpy(), atol=1e-11), name


def test_cp_selection_is_per_shard_and_ordered():
    """Each shard spends exactly S/P entries on its own tokens (a shard's high
    scores cannot take another shard's budget), and the concatenated
    sub-sequence is in (position, level) order over the whole sequence."""
    P = 4
    s = Shape(1, 1, 1024, 8, 4, 3, 128)
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((1, 1, 1024, 8)) for _ in range(3))
    q[:, :, :256] *= 10.0  # shard 0 has all the high norms; it still gets S/P entries only
    k[:, :, :256] *= 10.0
    f = oracle.cp_forward(s, q, k, v, P)
    n, sp = 1024 // P, 128 // P
    for r, part in enumerate(f["parts"]):
        assert part["idx"].shape[-1] == sp
        assert np.all((part["pos"] >= r * n) & (part["pos"] < (r + 1) * n))
    pos = f["pos"][0, 0]
    sh = f["shard"]
    offs = np.array([sh.level_off(l) for l in range(1, sh.L)])
    lev = np.concatenate([np.searchsorted(offs, part["idx"][0, 0], side="right") for part in f["parts"]])
    keys = pos.astype(np.int64) * 16 + lev
    assert np.all(np.diff(keys) > 0)
