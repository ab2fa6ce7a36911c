"""CUDA path vs the CPU oracle, stage by stage and fused, through the C ABI.

Tolerances (written here, used everywhere below):
  * scores, selected index sets, positions, slot map: bit-exact (integer
    results; both sides compute the scores in fp32 in the same fixed order);
  * pyramid levels (fp32 on the GPU, fp64 in the oracle): |err| <= 1e-5 |ref|
    + 1e-6 * rms(level);
  * gathered rows (fp16): within half an fp16 ulp of the fp64 value;
  * attention outputs and gradients: max-abs error <= 2e-2 and
    mean|err| / mean|ref| <= 1e-2 against the fp64 oracle.  A result the
    library stores in a 16-bit format cannot sit closer to the exact value
    than half an ulp of that format, so for those (and only those) the
    elementwise bound adds half an ulp: 2^-8 |ref| for bf16 results (the
    layer's O, dQ, dK, dV of bf16 workloads), 2^-11 |ref| for the fp16
    sub-sequence output os.  fp32 results (dqs, dks, dvs and every output of
    an fp32 workload) get the plain 2e-2.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from long_context_lh_b200 import lighthouse as lh
from long_context_lh_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


# half an ulp (relative) of the format a result is stored in
HALF_ULP = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 0.0}


def check_attn(got, ref, name, stored):
    """`stored`: the torch dtype the library wrote the result in."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bound = 2e-2 + HALF_ULP[stored] * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{name}: max err {err.max():.4g} at {worst} ref {ref[worst]:.4g}"
    scale = np.abs(ref).mean()
    if scale > 1e-6:  # a reference that is zero in exact arithmetic has no relative error
        rel = err.mean() / scale
        assert rel <= 1e-2, f"{name}: mean relative error {rel:.4g}"


def check_pyramid(got, ref, name):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    err = np.abs(got - ref)
    assert np.all(err <= 1e-5 * np.abs(ref) + 1e-6 * rms), f"{name}: max err {err.max():.3g}"


def check_gathered(got, ref):
    """fp16 rounding (half an ulp, <= 2^-11 relative; subnormals below 2^-14 have
    an absolute half-ulp of 2^-25) of an fp32 value within fp32 rounding of the
    fp64 pyramid value."""
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.abs(got - ref)
    bound = 2.0 ** -11 * np.abs(ref) + 2.0 ** -25 + 1e-6 * rms
    assert np.all(err <= bound), f"gather: max err {err.max():.3g}"


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def to_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def workload(name="tiny", **kw):
    return WORKLOADS[name].with_(**kw)


def oshape(w):
    return oracle.Shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)


def lshape(w):
    return lh.make_shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)


STAGE_CASES = [
    dict(),                                                   # tiny: fp32, p=4, L=3, S=512
    dict(dtype="bf16", dist="outliers"),
    dict(dtype="bf16", d=128, p=2, L=5, N=2048, S=640),
    dict(dtype="bf16", p=3, L=3, N=1152, S=200),              # non-power-of-two p, ragged S
    dict(dtype="bf16", L=1, N=1000, S=333),
    dict(dtype="bf16", p=2, L=2, N=256, S=384),               # S = M: everything selected
    dict(dtype="bf16", N=512, S=1),
    dict(dtype="bf16", p=4, L=5, N=2048, S=300),             # level 4 wider than a 64-row chunk
    dict(p=5, L=4, N=1000, S=100),                            # p^3 = 125 > 64, last chunk ragged
    dict(B=3, H=2, dtype="bf16", dist="outliers", N=2048, S=256),  # several batch rows
    # more units than clusters of 8 CTAs run at once: the selection takes smaller clusters
    dict(B=2, H=8, dtype="bf16", dist="outliers", N=4096, S=512),
    dict(B=2, H=12, dtype="bf16", N=4096, S=512),
]


def topk_both(shp, score, opt=None):
    """Both selection implementations (a thread-block cluster per unit without a
    workspace, device-wide passes with one) on the same scores: they must agree
    bit for bit; returns idx, pos, slot."""
    B, H, M = score.shape
    S_ = shp.S
    outs = []
    for with_ws in (False, True):
        idx = torch.full((B, H, S_), -7, dtype=torch.int32, device=DEV)
        pos = torch.full_like(idx, -7)
        slot = torch.full((B, H, M), -7, dtype=torch.int32, device=DEV)
        ws, wsb = None, 0
        if with_ws:
            wsb = lh.lh_topk_workspace_bytes(shp)
            ws = torch.full((wsb,), 0x5A, dtype=torch.uint8, device=DEV)  # garbage: zeroed by the call
        if opt is None:
            lh.lh_topk_select(shp, score, idx, pos, slot, ws, wsb)
        else:
            lh.lh_topk_select_ex(shp, score, idx, pos, slot, opt, ws, wsb)
        outs.append((idx, pos, slot))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b), "cluster and pass selections differ"
    return outs[1]


def run_front(w, x):
    """GPU pyramid, score and selection for inputs x (device tensors)."""
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    M = lh.lh_num_entries(shp)
    U = w.B * w.H
    pyr = [torch.zeros((w.B, w.H, max(M - w.N, 1), w.d), dtype=torch.float32, device=DEV)
           for _ in range(3)]
    score = torch.zeros((w.B, w.H, M), dtype=torch.float32, device=DEV)
    lh.lh_build_pyramid(shp, dt, x["q"], x["k"], x["v"], *pyr)
    lh.lh_score(shp, dt, x["q"], x["k"], score)
    idx, pos, slot = topk_both(shp, score)
    del U
    return pyr, score, idx, pos, slot


@pytest.mark.parametrize("case", STAGE_CASES, ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()) or "tiny")
def test_front_stages_match_oracle(case):
    w = workload(**case)
    xc = make_inputs(w, "cpu", with_dO=False)
    x = to_dev(xc)
    pyr, score, idx, pos, slot = run_front(w, x)
    s = oshape(w)
    qf, kf, vf = (xc[n].float().numpy() for n in ("q", "k", "v"))
    sc_ref = oracle.score(s, qf, kf)
    assert np.array_equal(score.cpu().numpy(), sc_ref), "scores differ in some bit"
    i_ref, p_ref, s_ref = oracle.select(s, sc_ref)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(pos.cpu().numpy(), p_ref)
    assert np.array_equal(slot.cpu().numpy(), s_ref)
    if w.L > 1:
        for t, ref in zip(pyr, (oracle.pyramid(s, a) for a in (qf, kf, vf))):
            check_pyramid(t.cpu().numpy(), ref, "pyramid")


@pytest.mark.parametrize("case", [dict(N=524288, L=2, S=3000), dict(N=262144, p=2, L=3, S=100000)],
                         ids=str)
def test_topk_on_large_units_matches_oracle(case):
    """The first case (more than 2^19 entries per unit) takes the 16-CTA cluster
    where the device allows it, with the keys cached in shared memory; the second
    has too many keys per CTA for the cache and reads them from L2 in each pass.
    The selection must be exact either way."""
    w = workload(dtype="bf16", dist="outliers", H=2, **case)
    xc = make_inputs(w, "cpu", with_dO=False)
    x = to_dev(xc)
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    M = lh.lh_num_entries(shp)
    score = torch.zeros((w.B, w.H, M), dtype=torch.float32, device=DEV)
    lh.lh_score(shp, dt, x["q"], x["k"], score)
    idx, pos, slot = topk_both(shp, score)
    s = oshape(w)
    sc_ref = oracle.score(s, xc["q"].float().numpy(), xc["k"].float().numpy())
    assert np.array_equal(score.cpu().numpy(), sc_ref), "scores differ in some bit"
    i_ref, p_ref, s_ref = oracle.select(s, sc_ref)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(pos.cpu().numpy(), p_ref)
    assert np.array_equal(slot.cpu().numpy(), s_ref)


@pytest.mark.parametrize("N,S,L", [(2048, 300, 3), (32768, 3000, 2)], ids=["list", "beyond-list"])
def test_ties_beyond_inheritance_are_broken_by_gid(N, S, L):
    """Quantised inputs make many equal scores; the radix select on gids must agree.
    The second case has thousands of entries tied at the threshold, more than the
    pass selection resolves from a list (it then runs radix passes over the gids)."""
    w = workload(dtype="bf16", N=N, S=S, L=L, H=3)
    xc = make_inputs(w, "cpu", with_dO=False)
    for n in ("q", "k"):
        xc[n] = (xc[n].float() * 0).to(torch.bfloat16)
        xc[n][..., 0] = torch.randint(0, 3, xc[n].shape[:-1]).to(torch.bfloat16)
    x = to_dev(xc)
    _, score, idx, pos, slot = run_front(w, x)
    s = oshape(w)
    sc_ref = oracle.score(s, xc["q"].float().numpy(), xc["k"].float().numpy())
    assert np.array_equal(score.cpu().numpy(), sc_ref)
    i_ref, p_ref, s_ref = oracle.select(s, sc_ref)
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(slot.cpu().numpy(), s_ref)


def gpu_gather(w, x, pyr, idx):
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    out = [torch.empty((w.B, w.H, w.S, w.d), dtype=torch.float16, device=DEV) for _ in range(3)]
    lh.lh_gather(shp, dt, x["q"], x["k"], x["v"], *pyr, idx, *out)
    return out


def scatter_f32(s, os_, slot):
    """Scatter-back restated in fp32, the kernel's precision: per token, the rows
    of its selected entries summed in ascending level order, then one IEEE
    division by their count (zero when none).  The fp32 output must equal it
    value for value."""
    os_ = np.asarray(os_, np.float32)
    t = np.arange(s.N)
    acc = np.zeros((s.B, s.H, s.N, s.d), np.float32)
    cnt = np.zeros((s.B, s.H, s.N), np.int64)
    for l in range(s.L):
        sl = slot[:, :, s.level_off(l) + t // s.p ** l]
        sel = sl >= 0
        rows = np.take_along_axis(os_, np.maximum(sl, 0)[..., None], axis=2)
        acc = acc + np.where(sel[..., None], rows, np.float32(0))
        cnt += sel
    div = np.maximum(cnt, 1).astype(np.float32)[..., None]
    return np.where(cnt[..., None] > 0, acc / div, np.float32(0)), cnt


GS_CASES = STAGE_CASES[:4] + [
    STAGE_CASES[8],
    dict(p=2, L=8, N=1024, S=600),
    dict(dtype="bf16", p=4, L=2, N=1000, S=256),   # N not a multiple of p^2: ragged last thread
    dict(dtype="bf16", p=2, L=2, N=1002, S=384),
    dict(dtype="bf16", d=128, p=4, L=4, N=4096, S=512),
    dict(p=4, L=5, N=2048, S=384),                 # fp32 input, several batches per span walk
]


@pytest.mark.parametrize("case", GS_CASES, ids=str)
def test_gather_and_scatter_match_oracle(case):
    w = workload(**case)
    xc = make_inputs(w, "cpu")
    x = to_dev(xc)
    pyr, score, idx, pos, slot = run_front(w, x)
    qs, ks, vs = gpu_gather(w, x, pyr, idx)
    s = oshape(w)
    i_ref = idx.cpu().numpy()
    for t, n in zip((qs, ks, vs), ("q", "k", "v")):
        a = xc[n].float().numpy()
        ref = oracle.gather(s, a, oracle.pyramid(s, a), i_ref)
        check_gathered(f64(t), ref)
    # scatter-back of arbitrary bf16 rows
    os_ = torch.randn((w.B, w.H, w.S, w.d), device=DEV).to(torch.float16)
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=x["q"].dtype, device=DEV)
    ic = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=DEV)
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    lh.lh_scatter_back(shp, dt, os_, slot, o, ic)
    ref = oracle.scatter(s, f64(os_), slot.cpu().numpy())
    tol = 2.0 ** -8 if w.dtype == "bf16" else 1e-6
    assert np.all(np.abs(f64(o) - ref) <= tol * np.abs(ref) + 1e-6)  # output-dtype rounding
    if w.dtype == "f32":  # the correctly rounded fp32 quotient, for every count that occurs
        exact, cnt = scatter_f32(s, f64(os_), slot.cpu().numpy())
        got = o.cpu().numpy()
        assert np.all(got == exact), f"scatter: {np.count_nonzero(got != exact)} values differ"
        if w.L == 8:  # counts 2..8 all occur in this draw
            assert set(np.unique(cnt)) >= set(range(2, 9))
        icg = ic.cpu().numpy()
        assert np.array_equal(icg, np.where(cnt > 0, np.float32(1) / np.maximum(cnt, 1).astype(np.float32), 0))
    # scatter-back adjoint, with and without the saved counts
    dO = x["dO"]
    for use_ic in (True, False):
        dos = torch.empty((w.B, w.H, w.S, w.d), dtype=torch.float16, device=DEV)
        lh.lh_scatter_back_bwd(shp, dt, dO, slot, ic if use_ic else None, dos)
        ref = oracle.scatter_bwd(s, f64(dO), idx.cpu().numpy(), slot.cpu().numpy())
        got = f64(dos)
        assert np.all(np.abs(got - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-5 * (1 + np.abs(ref).max()))
    # gather adjoint
    d3 = [torch.randn((w.B, w.H, w.S, w.d), device=DEV) for _ in range(3)]
    dx = [torch.empty((w.B, w.H, w.N, w.d), dtype=x["q"].dtype, device=DEV) for _ in range(3)]
    lh.lh_gather_bwd(shp, dt, *d3, slot, *dx)
    for a, b in zip(d3, dx):
        ref = oracle.gather_bwd(s, f64(a), slot.cpu().numpy())
        assert np.all(np.abs(f64(b) - ref) <= tol * np.abs(ref) + 1e-6)


@pytest.mark.parametrize("case", STAGE_CASES, ids=str)
def test_pooled_gather_equals_pyramid_gather_bitwise(case):
    """lh_gather_pooled (no pyramid in HBM) == lh_gather on lh_build_pyramid, bit for bit."""
    w = workload(**case)
    x = to_dev(make_inputs(w, "cpu", with_dO=False))
    pyr, score, idx, pos, slot = run_front(w, x)
    a = gpu_gather(w, x, pyr, idx)
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    b = [torch.empty_like(t) for t in a]
    lh.lh_gather_pooled(shp, dt, x["q"], x["k"], x["v"], idx, *b)
    torch.cuda.synchronize()
    for ta, tb in zip(a, b):
        assert torch.equal(ta, tb)


ATTN_CASES = [(2, 512, 64), (1, 1000, 64), (1, 1, 64), (2, 384, 128), (1, 200, 128)]


@pytest.mark.parametrize("impl", [0, 1], ids=["tcgen05", "mma_sync"])
@pytest.mark.parametrize("U,S,d", ATTN_CASES)
def test_attention_matches_oracle(U, S, d, impl):
    prev = lh.lh_set_attention_impl(impl)
    try:
        g = torch.Generator().manual_seed(100 + S + d)
        qs, ks, vs, dos = (torch.randn((1, U, S, d), generator=g).mul(1.5).to(torch.float16)
                           for _ in range(4))
        shp = lh.make_shape(1, U, max(S, 1), d, 2, 1, S)
        qd, kd, vd, dod = (t.to(DEV) for t in (qs, ks, vs, dos))
        os_ = torch.empty_like(qd)
        lse = torch.empty((1, U, S), dtype=torch.float32, device=DEV)
        lh.lh_subseq_attn_fwd(shp, qd, kd, vd, 0.0, os_, lse)
        s = oracle.Shape(1, U, max(S, 1), d, 2, 1, S)
        sc = 1.0 / np.sqrt(d)
        o_ref, lse_ref = oracle.attn_fwd(s, f64(qs), f64(ks), f64(vs), sc)
        check_attn(f64(os_), o_ref, "os", os_.dtype)
        assert np.abs(f64(lse) - lse_ref).max() < 2e-2
        dq, dk, dv = (torch.empty((1, U, S, d), dtype=torch.float32, device=DEV) for _ in range(3))
        wsb = lh.lh_attn_bwd_workspace_bytes(shp)
        ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
        lh.lh_subseq_attn_bwd(shp, qd, kd, vd, os_, lse, dod, 0.0, dq, dk, dv, ws, wsb)
        refs = oracle.attn_bwd(s, f64(qs), f64(ks), f64(vs), f64(dos), sc)
        for name, got, ref in zip(("dqs", "dks", "dvs"), (dq, dk, dv), refs):
            check_attn(f64(got), ref, name, got.dtype)
        assert lh.lh_read_device_status() == 0
    finally:
        lh.lh_set_attention_impl(prev)


@pytest.mark.parametrize("case", [dict(), dict(dtype="bf16", dist="outliers", N=8192, S=1024, L=4),
                                  dict(dtype="bf16", d=128, p=2, L=4, N=2048, S=500),
                                  # several batch rows: units are (batch, head) pairs
                                  dict(B=2, H=3, dtype="bf16", dist="outliers", N=4096, S=512, L=3),
                                  dict(B=2, H=1, dtype="bf16", dist="lognormal", d=128, N=4096, S=640,
                                       L=4)], ids=str)
def test_fused_forward_backward_match_oracle(case):
    w = workload(**case)
    xc = make_inputs(w, "cpu")
    x = to_dev(xc)
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    dq, dk, dv = lh.backward(saved, x["dO"])
    torch.cuda.synchronize()
    s = oshape(w)
    f = [xc[n].float().numpy() for n in ("q", "k", "v", "dO")]
    ref = oracle.forward(s, *f[:3])
    sv = lambda which: lh.saved_view(saved.shape, saved.buf, which).cpu().numpy()
    assert np.array_equal(sv(lh.SAVED_IDX), ref["idx"])
    assert np.array_equal(sv(lh.SAVED_POS), ref["pos"])
    assert np.array_equal(sv(lh.SAVED_SLOT), ref["slot"])
    check_attn(f64(o), ref["o"], "o", o.dtype)
    bref = oracle.backward(s, ref, f[3])
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_attn(f64(t), bref[name], name, t.dtype)


VARIANT_CASES = [
    dict(score_mode=1, keep=False, w=dict(dtype="bf16", dist="outliers")),
    dict(score_mode=2, keep=False, w=dict(dtype="bf16", d=128, p=2, L=5, N=2048, S=640)),
    dict(score_mode=0, keep=True, w=dict(dtype="bf16", N=4096, L=4, S=300)),   # 64 coarsest of 300
    dict(score_mode=2, keep=True, w=dict(p=3, L=3, N=1152, S=200)),            # fp32, generic p
    dict(score_mode=1, keep=True, w=dict(dtype="bf16", p=4, L=2, N=1024, S=256)),  # S = n_{L-1}
    dict(score_mode=0, keep=True, w=dict(dtype="bf16", dist="outliers", H=2, N=524288, L=5, S=4096)),
    dict(score_mode=0, keep=False, scatter=1, w=dict(dtype="bf16", dist="outliers")),      # sum
    dict(score_mode=0, keep=False, scatter=2, w=dict(dtype="bf16", dist="outliers")),      # last token
    dict(score_mode=2, keep=True, scatter=2, w=dict(p=3, L=3, N=1152, S=200)),
    dict(score_mode=0, keep=False, scatter=1, w=dict(dtype="bf16", d=128, p=2, L=5, N=2048, S=640)),
]


@pytest.mark.parametrize("case", VARIANT_CASES, ids=str)
def test_variant_stages_match_oracle(case):
    """Score ablations and keep-coarsest through the _ex stage calls: scores and
    the selection bit-exact against the oracle with the same options."""
    w = workload(**case["w"])
    opt = lh.make_options(case["keep"], case["score_mode"])
    xc = make_inputs(w, "cpu", with_dO=False)
    x = to_dev(xc)
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    M = lh.lh_num_entries(shp)
    score = torch.zeros((w.B, w.H, M), dtype=torch.float32, device=DEV)
    score2 = torch.zeros_like(score)
    pyr = [torch.zeros((w.B, w.H, max(M - w.N, 1), w.d), dtype=torch.float32, device=DEV)
           for _ in range(3)]
    lh.lh_score_ex(shp, dt, x["q"], x["k"], score, opt)
    lh.lh_build_pyramid_score_ex(shp, dt, x["q"], x["k"], x["v"], *pyr, score2, opt)
    idx, pos, slot = topk_both(shp, score, opt)
    torch.cuda.synchronize()
    s = oshape(w)
    sc_ref = oracle.score(s, xc["q"].float().numpy(), xc["k"].float().numpy(), mode=case["score_mode"])
    assert np.array_equal(score.cpu().numpy(), sc_ref), "scores differ in some bit"
    assert np.array_equal(score2.cpu().numpy(), sc_ref), "fused pass: scores differ"
    i_ref, p_ref, s_ref = oracle.select(s, sc_ref, keep_coarsest=case["keep"])
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(pos.cpu().numpy(), p_ref)
    assert np.array_equal(slot.cpu().numpy(), s_ref)


@pytest.mark.parametrize("case", VARIANT_CASES[:4] + VARIANT_CASES[6:], ids=str)
def test_variant_forward_backward_match_oracle(case):
    """lh_forward_ex (+ lh_backward_ex on its saved selection) against the oracle
    pipeline with the same options."""
    w = workload(**case["w"])
    opt = lh.make_options(case["keep"], case["score_mode"], case.get("scatter", 0))
    xc = make_inputs(w, "cpu")
    x = to_dev(xc)
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S, options=opt)
    dq, dk, dv = lh.backward(saved, x["dO"])
    torch.cuda.synchronize()
    s = oshape(w)
    f = [xc[n].float().numpy() for n in ("q", "k", "v", "dO")]
    ref = oracle.forward(s, *f[:3], score_mode=case["score_mode"], keep_coarsest=case["keep"],
                         scatter_mode=case.get("scatter", 0))
    sv = lambda which: lh.saved_view(saved.shape, saved.buf, which).cpu().numpy()
    assert np.array_equal(sv(lh.SAVED_IDX), ref["idx"])
    assert np.array_equal(sv(lh.SAVED_SLOT), ref["slot"])
    check_attn(f64(o), ref["o"], "o", o.dtype)
    bref = oracle.backward(s, ref, f[3])
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_attn(f64(t), bref[name], name, t.dtype)
    if case["keep"] and case.get("scatter", 0) != 2:  # every token has a contributor
        assert np.all(sv(lh.SAVED_INV_COUNT) > 0)


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("case", [GS_CASES[1], GS_CASES[3], GS_CASES[5]], ids=str)
def test_scatter_modes_match_oracle(case, mode):
    """The scatter ablations (sum, last token) and their adjoints through the
    _ex stage calls, with and without the saved weights, against the oracle."""
    w = workload(**case)
    x = to_dev(make_inputs(w, "cpu"))
    _, _, idx, _, slot = run_front(w, x)
    opt = lh.make_options(False, 0, mode)
    shp, dt = lshape(w), lh.dtype_code(x["q"].dtype)
    s = oshape(w)
    os_ = torch.randn((w.B, w.H, w.S, w.d), device=DEV).to(torch.float16)
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=x["q"].dtype, device=DEV)
    ic = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=DEV)
    lh.lh_scatter_back_ex(shp, dt, os_, slot, o, ic, opt)
    ref = oracle.scatter(s, f64(os_), slot.cpu().numpy(), mode)
    tol = 2.0 ** -8 if w.dtype == "bf16" else 1e-6
    assert np.all(np.abs(f64(o) - ref) <= tol * np.abs(ref) + 1e-6)
    for use_ic in (True, False):
        dos = torch.empty((w.B, w.H, w.S, w.d), dtype=torch.float16, device=DEV)
        lh.lh_scatter_back_bwd_ex(shp, dt, x["dO"], slot, ic if use_ic else None, dos, opt)
        ref = oracle.scatter_bwd(s, f64(x["dO"]), idx.cpu().numpy(), slot.cpu().numpy(), mode)
        assert np.all(np.abs(f64(dos) - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-5 * (1 + np.abs(ref).max()))


def test_variant_options_rejected_on_the_host():
    w = workload(dtype="bf16", N=4096, L=3, S=128)   # 256 coarsest entries > S
    shp = lshape(w)
    assert lh.lh_validate_options(shp, lh.make_options(True)) == lh.LH_ERR_SHAPE
    assert lh.lh_validate_options(shp, lh.make_options(False, 7)) == lh.LH_ERR_INVALID_ARG
    bad = lh.make_options(False)
    bad.reserved = 1
    assert lh.lh_validate_options(shp, bad) == lh.LH_ERR_INVALID_ARG
    assert lh.lh_validate_options(shp, lh.make_options(False, 0, 3)) == lh.LH_ERR_INVALID_ARG
    x = to_dev(make_inputs(w, "cpu", with_dO=False))
    with pytest.raises(lh.LighthouseError):
        lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S, options=lh.make_options(True))


def test_degenerate_L1_full_selection_equals_causal_sdpa():
    w = workload(dtype="bf16", L=1, N=512, S=512, H=2)
    xc = make_inputs(w, "cpu")
    x = to_dev(xc)
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    assert torch.equal(lh.saved_view(saved.shape, saved.buf, lh.SAVED_IDX)[0, 0].cpu(),
                       torch.arange(512, dtype=torch.int32))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(xc[n].double() for n in ("q", "k", "v")), is_causal=True)
    check_attn(f64(o), ref.numpy(), "o", o.dtype)


def test_bitwise_deterministic():
    w = workload(dtype="bf16", dist="outliers", N=8192, S=1024, L=4, H=4)
    x = to_dev(make_inputs(w, "cpu"))
    outs = []
    for _ in range(2):
        o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
        grads = lh.backward(saved, x["dO"])
        outs.append([o.clone(), saved.buf.clone(), *[g.clone() for g in grads]])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def check_full_size(name, device_draw=False, n_tokens=24, full_backward_head0=False):
    """A benchmark workload at full size, through lh_forward / lh_backward as the
    bench launches them.

    Every head: scores and the selection (idx, slot) bit-exact.  Heads 0 and
    H-1: gathered rows; the contributor slots R of n_tokens random tokens (plus
    tokens without contributors): attention rows os[R] from the oracle, and the
    layer's outputs O, dQ, dK, dV at those tokens, each built by the oracle's own
    scatter-back / gather adjoint from the oracle's rows R (oracle.scatter_bwd
    for dos, oracle.attn_bwd_sampled for the gradient rows and columns).  No
    oracle input comes from the GPU: the selection it uses is its own (checked
    equal first)."""
    w = WORKLOADS[name]
    xg = make_inputs(w, "cuda" if device_draw else "cpu")
    x = to_dev(xg)
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    dq, dk, dv = lh.backward(saved, x["dO"])
    torch.cuda.synchronize()
    sv = lambda which: lh.saved_view(saved.shape, saved.buf, which)
    idx_g, slot_g = sv(lh.SAVED_IDX).cpu().numpy(), sv(lh.SAVED_SLOT).cpu().numpy()
    s1 = oshape(w).unit()
    head = lambda t, h: t[:, h:h + 1].float().cpu().numpy()
    refs = {}
    for h in range(w.H):
        sc = oracle.score(s1, head(xg["q"], h), head(xg["k"], h))
        i_ref, _, s_ref = oracle.select(s1, sc)
        assert np.array_equal(idx_g[:, h:h + 1], i_ref), f"idx head {h}"
        assert np.array_equal(slot_g[:, h:h + 1], s_ref), f"slot head {h}"
        refs[h] = (i_ref, s_ref)
    rng = np.random.default_rng(7)
    scale = 1.0 / np.sqrt(w.d)
    for h in (0, w.H - 1):
        i_ref, s_ref = refs[h]
        xs = []
        for n in ("q", "k", "v"):
            a = head(xg[n], h)
            xs.append(oracle.gather(s1, a, oracle.pyramid(s1, a), i_ref))
        for ref, which in zip(xs, (lh.SAVED_QS, lh.SAVED_KS, lh.SAVED_VS)):
            check_gathered(f64(sv(which)[:, h:h + 1]), ref)
        slot_h = s_ref[0, 0]
        contrib = lambda t: [int(slot_h[s1.level_off(l) + t // w.p ** l]) for l in range(w.L)]
        toks, uncovered = [], []
        while len(toks) < n_tokens:
            t = int(rng.integers(w.N))
            (toks if any(z >= 0 for z in contrib(t)) else uncovered).append(t)
        rows = np.unique([z for t in toks for z in contrib(t) if z >= 0]).astype(np.int32)
        toks = np.array(toks + uncovered[:8], dtype=np.int64)
        os_r, _ = oracle.attn_fwd(s1, *xs, scale, rows=rows)
        check_attn(f64(sv(lh.SAVED_OS)[:, h:h + 1, rows]), os_r, f"os head {h}", torch.float16)
        os_part = np.zeros((1, 1, w.S, w.d))
        os_part[0, 0, rows] = os_r[0, 0]
        o_ref = oracle.scatter(s1, os_part, s_ref)[0, 0, toks]
        check_attn(f64(o[0, h, toks]), o_ref, f"o head {h}", o.dtype)
        dos_ref = oracle.scatter_bwd(s1, head(xg["dO"], h), i_ref, s_ref)
        g_r = oracle.attn_bwd_sampled(*(t[0, 0] for t in xs), dos_ref[0, 0], scale, rows)
        for gname, g_rows, got in zip(("dq", "dk", "dv"), g_r, (dq, dk, dv)):
            part = np.zeros((1, 1, w.S, w.d))
            part[0, 0, rows] = g_rows
            g_ref = oracle.gather_bwd(s1, part, s_ref)[0, 0, toks]
            check_attn(f64(got[0, h, toks]), g_ref, f"{gname} head {h}", got.dtype)
        if full_backward_head0 and h == 0:  # every token of head 0, from the full oracle backward
            full = oracle.attn_bwd(s1, *xs, dos_ref, scale)
            for gname, g_s, got in zip(("dq", "dk", "dv"), full, (dq, dk, dv)):
                check_attn(f64(got[:, :1]), oracle.gather_bwd(s1, g_s, s_ref), f"{gname} head 0 (all tokens)",
                           got.dtype)


def test_pretraining_shape_full_size():
    """The pretraining workload (H=16, N=98,304, S=8192), as the bench runs it; head 0's
    gradients at every token from the oracle's full attention backward."""
    check_full_size("pretrain", full_backward_head0=True)


def test_long_context_full_size():
    """The long-context workload (H=16, N=524,288, L=5, S=16,384), as the bench runs it."""
    check_full_size("long", device_draw=True)


def test_extreme_context_full_size():
    """The one-GPU extreme workload (H=8, N=1,048,576, d=128, L=6, S=16,384, log-normal
    token norms), as the bench runs it."""
    check_full_size("extreme", device_draw=True)


def test_attention_block_matches_oracle_chain():
    """The block (projections + Lighthouse + output projection, autograd) against
    the same chain with the attention and its backward taken from the oracle in
    fp64 and the projections applied by hand: the output and the gradients of the
    input and of both weight matrices."""
    from long_context_lh_b200.block import LighthouseBlock
    torch.manual_seed(3)
    B, N, H, d, p, L, S = 1, 2048, 2, 64, 4, 3, 384
    blk = LighthouseBlock(H * d, H, p, L, S, device=DEV)
    with torch.no_grad():
        for w in (blk.wqkv.weight, blk.wo.weight):
            w.copy_(torch.randn_like(w, dtype=torch.float32) / np.sqrt(H * d))
    x = torch.randn((B, N, H * d), device=DEV).to(torch.bfloat16).requires_grad_(True)
    g = torch.randn((B, N, H * d), device=DEV).to(torch.bfloat16)
    y = blk(x)
    y.backward(g)
    torch.cuda.synchronize()
    # the chain by hand, attention from the oracle (fp64); inputs to it from torch only
    s = oracle.Shape(B, H, N, d, p, L, S)
    with torch.no_grad():
        q, k, v = (t.float().cpu().numpy() for t in blk.split_heads(x))
        wo = f64(blk.wo.weight)
        wqkv = f64(blk.wqkv.weight)
    ref = oracle.forward(s, q, k, v)
    o = ref["o"]                                            # [B, H, N, d]
    o_flat = o.transpose(0, 2, 1, 3).reshape(B, N, H * d)
    y_ref = o_flat @ wo.T
    check_attn(f64(y), y_ref, "block output", y.dtype)
    gg = f64(g)
    dO = (gg @ wo).reshape(B, N, H, d).transpose(0, 2, 1, 3)
    bref = oracle.backward(s, ref, dO)
    dqkv = np.stack([bref["dq"], bref["dk"], bref["dv"]])   # [3, B, H, N, d]
    dqkv_flat = dqkv.transpose(1, 3, 0, 2, 4).reshape(B, N, 3 * H * d)
    x64 = f64(x)
    check_attn(f64(x.grad), dqkv_flat @ wqkv, "dx", x.grad.dtype)
    # The weight gradients are sums over all N tokens of (attention output or gradient)
    # x (input or upstream gradient): per-element attention errors within the bound
    # above accumulate like sqrt(N) in each entry, so these are checked in norm --
    # mean relative error <= 1e-2 (as every attention result) and the largest
    # error within 2% of the largest entry.
    for name, got, ref_w in (
            ("dWqkv", blk.wqkv.weight.grad, dqkv_flat.reshape(-1, 3 * H * d).T @ x64.reshape(-1, H * d)),
            ("dWo", blk.wo.weight.grad, gg.reshape(-1, H * d).T @ o_flat.reshape(-1, H * d))):
        err = np.abs(f64(got) - ref_w)
        assert err.mean() / np.abs(ref_w).mean() <= 1e-2, f"{name}: mean relative error"
        assert err.max() <= 2e-2 * np.abs(ref_w).max(), f"{name}: max err {err.max():.3g}"


def test_non_finite_inputs_complete_and_leave_the_context_usable():
    """Non-finite inputs give unspecified values but never an error, a hang or a
    device status: NaN and +-inf rows in q, k, v and dO (the selection works on
    key bits, every index it produces is in range, every loop has a fixed trip
    count).  A normal call afterwards still matches the oracle."""
    w = workload(dtype="bf16", N=4096, S=512, L=3, H=2)
    x = to_dev(make_inputs(w, "cpu"))
    for name, val, rows in (("q", float("nan"), (5, 77)), ("k", float("inf"), (100,)),
                            ("v", float("-inf"), (1000,)), ("dO", float("nan"), (3,))):
        for r in rows:
            x[name][0, 0, r, :8] = val
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    dq, dk, dv = lh.backward(saved, x["dO"])
    torch.cuda.synchronize()
    code = ctypes.c_uint32(0)
    assert lh._lib().lh_read_device_status(None, ctypes.byref(code)) == lh.LH_OK
    assert code.value == 0
    idx = lh.saved_view(saved.shape, saved.buf, lh.SAVED_IDX).cpu().numpy()
    assert idx.min() >= 0 and idx.max() < lh.lh_num_entries(saved.shape)
    # the context is healthy: a normal call still agrees with the oracle
    w2 = workload(dtype="bf16", N=2048, S=256, L=3, H=1)
    xc = make_inputs(w2, "cpu")
    x2 = to_dev(xc)
    o2, _ = lh.forward(x2["q"], x2["k"], x2["v"], w2.p, w2.L, w2.S)
    torch.cuda.synchronize()
    ref = oracle.forward(oshape(w2), *(xc[n].float().numpy() for n in ("q", "k", "v")))
    check_attn(f64(o2), ref["o"], "o after non-finite inputs", o2.dtype)


def test_finite_inputs_beyond_fp16_are_clipped_and_reported():
    """bf16 inputs may exceed the fp16 range of the sub-sequence.  The documented
    outcome: the selection is still exact (scores are fp32 from the inputs), the
    gathered rows are the oracle's rows clipped to +-65504, the attention output
    is the attention over those clipped fp16 rows, and lh_read_device_status
    reports LH_STATUS_FP16_SATURATED (once: reading clears it).

    Here the oracle's attention takes the clipped rows rounded to fp16 (on the
    CPU, from its own fp64 rows), i.e. exactly the operands the library defines
    the sub-sequence to hold: a logit of a 65504-sized row with a normal one
    moves by ~10 units when the normal row is rounded to fp16, which no
    attention tolerance absorbs, so unrounded operands would compare two
    different softmax distributions rather than two computations of one."""
    w = workload(dtype="bf16", N=4096, S=512, L=3, H=2)
    xc = make_inputs(w, "cpu")
    for name, tok, val in (("q", 1234, 1.0e5), ("k", 1234, -2.0e5), ("v", 1234, 3.0e5),
                           ("v", 77, 7.0e4), ("q", 3000, 9.0e4)):
        xc[name][0, 1, tok, ::3] = val   # head 1 only; head 0 stays in range
    assert torch.isfinite(xc["v"]).all()
    x = to_dev(xc)
    assert lh.lh_read_device_status() == 0
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    dq, dk, dv = lh.backward(saved, x["dO"])   # completes; values not compared
    torch.cuda.synchronize()
    code = lh.lh_read_device_status()
    assert code & lh.LH_STATUS_FP16_SATURATED, hex(code)
    assert code & ~lh.LH_STATUS_FP16_SATURATED == 0, hex(code)
    assert lh.lh_read_device_status() == 0  # cleared by the read
    sv = lambda which: lh.saved_view(saved.shape, saved.buf, which)
    s1 = oshape(w).unit()
    scale = 1.0 / np.sqrt(w.d)
    for h in range(w.H):
        head = lambda n: xc[n][:, h:h + 1].float().numpy()
        sc = oracle.score(s1, head("q"), head("k"))
        i_ref, _, s_ref = oracle.select(s1, sc)
        assert np.array_equal(sv(lh.SAVED_IDX)[:, h:h + 1].cpu().numpy(), i_ref), f"idx head {h}"
        xs = []
        for n, which in zip(("q", "k", "v"), (lh.SAVED_QS, lh.SAVED_KS, lh.SAVED_VS)):
            a = head(n)
            ref = np.clip(oracle.gather(s1, a, oracle.pyramid(s1, a), i_ref), -65504.0, 65504.0)
            check_gathered(f64(sv(which)[:, h:h + 1]), ref)
            xs.append(ref)
        if h == 1:
            assert np.abs(xs[2]).max() == 65504.0  # the clipped rows were selected
        xs = [a.astype(np.float16).astype(np.float64) for a in xs]
        os_r, _ = oracle.attn_fwd(s1, *xs, scale)
        check_attn(f64(sv(lh.SAVED_OS)[:, h:h + 1]), os_r, f"os head {h}", torch.float16)
    # a call with inputs in range afterwards reports nothing
    x2 = to_dev(make_inputs(w, "cpu"))
    lh.forward(x2["q"], x2["k"], x2["v"], w.p, w.L, w.S)
    assert lh.lh_read_device_status() == 0


def test_forward_pooled_path_matches_oracle_and_pyramid_stages():
    """A small budget over a long input makes lh_forward gather pooled rows (no
    pyramid level written).  Its selection and output must match the oracle, and
    its gathered rows must be bitwise those of the pyramid stage path."""
    w = workload(dtype="bf16", dist="outliers", N=65536, S=256, L=3, H=2)
    shp = lshape(w)
    assert lh.lh_forward_gather_path(shp, lh.LH_BF16) == 1
    xc = make_inputs(w, "cpu")
    x = to_dev(xc)
    o, saved = lh.forward(x["q"], x["k"], x["v"], w.p, w.L, w.S)
    dq, dk, dv = lh.backward(saved, x["dO"])
    torch.cuda.synchronize()
    sv = lambda which: lh.saved_view(saved.shape, saved.buf, which)
    s = oshape(w)
    f = [xc[n].float().numpy() for n in ("q", "k", "v", "dO")]
    ref = oracle.forward(s, *f[:3])
    assert np.array_equal(sv(lh.SAVED_IDX).cpu().numpy(), ref["idx"])
    check_attn(f64(o), ref["o"], "o", o.dtype)
    bref = oracle.backward(s, ref, f[3])
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_attn(f64(t), bref[name], name, t.dtype)
    # the pyramid stage path on the same selection gives the same rows, bit for bit
    M = lh.lh_num_entries(shp)
    pyr = [torch.empty((w.B, w.H, M - w.N, w.d), dtype=torch.float32, device=DEV) for _ in range(3)]
    lh.lh_build_pyramid(shp, lh.LH_BF16, x["q"], x["k"], x["v"], *pyr)
    rows = [torch.empty((w.B, w.H, w.S, w.d), dtype=torch.float16, device=DEV) for _ in range(3)]
    lh.lh_gather(shp, lh.LH_BF16, x["q"], x["k"], x["v"], *pyr, sv(lh.SAVED_IDX), *rows)
    torch.cuda.synchronize()
    for got, which in zip(rows, (lh.SAVED_QS, lh.SAVED_KS, lh.SAVED_VS)):
        assert torch.equal(got, sv(which))
