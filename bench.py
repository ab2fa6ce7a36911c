"""Benchmark of one Lighthouse Attention layer (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload pretrain|long|extreme] [--attn tc|mma] [--no-cpu] [--no-dense]

A step is one pass of the whole hot path over one batch of synthetic input:
pyramid + scores (one pass over Q, K, V), joint top-S, gather, causal
sub-sequence attention, scatter-back, then the backward through scatter-back,
attention and gather.
The default workload is the pretraining shape (B=1, H=16, N=98,304, d=64,
p=4, L=4, S=8192, bf16, 1% high-norm outlier tokens).  Inputs (3 x 201 MB plus
dO) are larger than the 126 MB L2, so no flush is needed between steps.

Rank 0 prints one JSON line.  With torchrun (N > 1) every rank runs its own
independent copy of the workload (heads are independent: weak scaling, no
collective on the data path); the step time is the max over ranks.
`--impl reference` times the CPU oracle on this host instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_lh_b200 import replicas  # noqa: E402
from long_context_lh_b200.synth import WORKLOADS, make_inputs  # noqa: E402

METRIC = "Lighthouse layer tokens/s fwd & fwd+bwd at N=98K/512K; % of HBM/TC roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + written) per launch of each stage, from one ncu capture of
# the full-size pretraining workload (the committed launch-list capture, with
# dram__bytes_read.sum and dram__bytes_write.sum, one pass).  Each entry
# carries a hash of the sources its kernels are built from; when they no longer
# match, the kernel has changed since the counters were taken and the traffic is
# reported as null.  Writes still in L2 when a kernel ends are counted by the
# kernel that evicts them, so a stage that writes more than L2 holds reads low.
MEASURED_TRAFFIC = {  # workload: {stage: (bytes per launch, sources, sha1[:16])}
    "pretrain": {
        "pyramid_score": (9.6650e+08, ('k_pyramid.cu', 'lh_internal.cuh'), "faf8e790685b35eb"),
        "topk": (4.7600e+07, ('k_topk.cu', 'lh_internal.cuh'), "61533dd39326a401"),
        "gather": (9.8800e+07, ('k_gather_scatter.cu', 'lh_internal.cuh'), "3db08f39fc50e30c"),
        "scatter": (1.6990e+08, ('k_gather_scatter.cu', 'lh_internal.cuh'), "3db08f39fc50e30c"),
        "scatter_bwd": (2.2560e+08, ('k_gather_scatter.cu', 'lh_internal.cuh'), "3db08f39fc50e30c"),
        "gather_bwd": (6.5840e+08, ('k_gather_scatter.cu', 'lh_internal.cuh'), "3db08f39fc50e30c"),
        "attn_fwd": (5.0400e+07, ('k_attn_tc.cu', 'tc_common.cuh', 'lh_internal.cuh'), "c4abb2f38acc8eb9"),
        "attn_bwd": (1.9460e+08, ('k_attn_tc.cu', 'tc_common.cuh', 'k_gather_scatter.cu', 'lh_internal.cuh'), "66ab60581431953c"),
    },
}


def measured_traffic(workload: str, stage: str):
    """DRAM bytes per launch of the stage, or None when unmeasured or stale."""
    import hashlib
    ent = MEASURED_TRAFFIC.get(workload, {}).get(stage)
    if ent is None:
        return None
    nbytes, srcs, sha = ent
    d = hashlib.sha1()
    for f in srcs:
        with open(os.path.join(ROOT, "long_context_lh_b200", "csrc", f), "rb") as fh:
            d.update(fh.read())
    return nbytes if d.hexdigest()[:16] == sha else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------ algorithmic work
def algorithmic(w, span_rows=None):
    """Algorithmic bytes / FLOPs per stage for one step (whole job on one GPU).

    Bytes count each tensor the stage must read or write once (inputs in the
    workload dtype, gathered rows fp16, sub-sequence gradients fp32); FLOPs
    count the causal attention products only.  The pooled gather must read, for
    every selected entry, the p^l level-0 rows its pooled value is the mean of
    (`span_rows`, summed over units, from the actual selection)."""
    U, N, d, S, M = w.B * w.H, w.N, w.d, w.S, w.M
    es = 2 if w.dtype == "bf16" else 4
    E = N * d
    span_rows = U * S if span_rows is None else span_rows
    R = (M - N) / N
    return {
        "pyramid_score": U * (3 * E * es + 12 * E * R + 4 * M),
        "score": U * (2 * E * es + 4 * M),
        "topk": U * (4 * M + 4 * M + 8 * S),
        "gather": U * (4 * S + S * 3 * d * (4 + 2)),
        "gather_pooled": U * 4 * S + span_rows * 3 * d * es + U * S * 3 * d * 2,
        "attn_fwd_flop": U * 2.0 * S * S * d,
        "scatter": U * (4 * M + S * d * 2 + E * es + 4 * N),
        "scatter_bwd": U * (E * es + 4 * N + 4 * M + S * d * 2),
        "attn_bwd_flop": U * 5.0 * S * S * d,
        "gather_bwd": U * (4 * M + 3 * S * d * 4 + 3 * E * es),
    }


# --------------------------------------------------------------------- clocks
class NvmlClockSampler:
    """SM clock and throttle reasons of this process's GPU every ~2 ms through NVML
    (read only), so that a timed region of a few tens of milliseconds has samples;
    `window` marks the timed region (host clock) and the summary keeps the
    samples inside it."""
    HW_SLOWDOWN, SW_POWER_CAP, SW_THERMAL, HW_THERMAL = 0x8, 0x4, 0x20, 0x40

    def __init__(self, device: torch.device):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(device)
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        self.max = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples, self.windows, self.stop = [], [], False

    def __enter__(self):
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def _run(self):
        nv = self.nv
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = self.reasons_fn(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def __exit__(self, *a):
        self.stop = True
        self.thread.join(timeout=1)

    def summary(self):
        inside = [smp for smp in self.samples if any(a <= smp[0] <= b for a, b in self.windows)]
        reasons = set()
        for _, _, rs in inside:
            for bit, name in ((self.HW_SLOWDOWN, "hw_slowdown"), (self.HW_THERMAL, "hw_thermal_slowdown"),
                              (self.SW_THERMAL, "sw_thermal_slowdown"), (self.SW_POWER_CAP, "sw_power_cap")):
                if rs & bit:
                    reasons.add(name)
        sm = [smp[1] for smp in inside]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(self.max),
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, every 2 ms"}


def clock_sampler(local_rank: int, device: torch.device):
    """The NVML sampler, or nvidia-smi's 50 ms loop where NVML is unavailable."""
    try:
        return NvmlClockSampler(device)
    except Exception:
        return ClockSampler(local_rank)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def window(self, t0, t1):
        pass

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ our arm
STAGES_FWD = ["pyramid_score", "topk", "gather", "attn_fwd", "scatter"]
STAGES_BWD = ["scatter_bwd", "attn_bwd", "gather_bwd"]


def measure(lh, w, args, rk, dev, peaks, steps, warmup, backward=True, batch=0, clocks=False):
    """Time one workload through lh_forward (+ lh_backward) on this rank's GPU, then
    replay the same launches stage by stage with events between stages.  Returns
    the timings, the per-stage roofline report, the tensors of the fused run and
    the peak device memory the fused path held (inputs, outputs, saved state and
    workspace)."""
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    mem0 = torch.cuda.memory_allocated(dev)
    shp = lh.make_shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)
    dt = lh.dtype_code(w.torch_dtype)
    x = make_inputs(w, dev, with_dO=backward, batch=batch)  # each rank: its own batch
    q, k, v = x["q"], x["k"], x["v"]
    dO = x.get("dO")
    o = torch.empty_like(q)
    dq, dk, dv = ((torch.empty_like(q) for _ in range(3)) if backward else (None, None, None))
    saved = torch.empty(lh.lh_saved_bytes(shp), dtype=torch.uint8, device=dev)
    wsb = lh.lh_workspace_bytes(shp, dt, backward)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream

    def fwd_only():
        lh.lh_forward(shp, dt, q, k, v, 0.0, o, saved, ws, wsb, sp)

    def step():
        fwd_only()
        if backward:
            lh.lh_backward(shp, dt, saved, dO, 0.0, dq, dk, dv, ws, wsb, sp)

    def timed(fn, K, clk=None):
        """Device time of K calls on this rank; the max over ranks is returned."""
        replicas.barrier(rk)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if clk is not None:
            clk.window(h0, time.perf_counter())
        ms = e0.elapsed_time(e1)
        replicas.barrier(rk)
        return replicas.max_over_ranks(rk, ms, dev)

    clk = clock_sampler(rk.local_rank, dev) if clocks else None
    with torch.cuda.stream(stream):
        if clk:
            clk.__enter__()  # sampling from the warm-up on; the summary keeps the timed region
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        status = lh.lh_read_device_status(stream)
        if clk:
            try:
                ms_step = timed(step, steps, clk) / steps
            finally:
                clk.__exit__(None, None, None)
        else:
            ms_step = timed(step, steps) / steps
        ms_fwd = timed(fwd_only, steps) / steps if backward else ms_step
    torch.cuda.synchronize()
    peak_bytes = torch.cuda.max_memory_allocated(dev) - mem0

    # stage-by-stage replica of the same launches, for per-kernel durations
    M, U = w.M, w.B * w.H
    stages = STAGES_FWD + (STAGES_BWD if backward else [])

    def view(which, dtype, n):
        off = lh.lh_saved_offset(shp, which)
        return saved[off:off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    idx = view(lh.SAVED_IDX, torch.int32, U * w.S)
    pos = view(lh.SAVED_POS, torch.int32, U * w.S)
    slot = view(lh.SAVED_SLOT, torch.int32, U * M)
    qs, ks, vs, os_ = (view(i, torch.float16, U * w.S * w.d)
                       for i in (lh.SAVED_QS, lh.SAVED_KS, lh.SAVED_VS, lh.SAVED_OS))
    lse = view(lh.SAVED_LSE, torch.float32, U * w.S)
    ic = view(lh.SAVED_INV_COUNT, torch.float32, U * w.N)
    npyr = max(U * (M - w.N) * w.d, 1)
    pq, pk, pv = (torch.empty(npyr, dtype=torch.float32, device=dev) for _ in range(3))
    score = torch.empty(U * M, dtype=torch.float32, device=dev)
    # the selection as lh_forward runs it: device-wide passes (with a workspace) or
    # one cluster per unit (without)
    tbw = lh.lh_topk_workspace_bytes(shp) if lh.lh_forward_topk_path(shp) == 1 else 0
    tws = torch.empty(tbw, dtype=torch.uint8, device=dev) if tbw else None
    if backward:
        dos = torch.empty(U * w.S * w.d, dtype=torch.float16, device=dev)
        dqs, dks, dvs = (torch.empty(U * w.S * w.d, dtype=torch.float32, device=dev) for _ in range(3))
        abw = lh.lh_attn_bwd_workspace_bytes(shp)
        aws = torch.empty(abw, dtype=torch.uint8, device=dev)

    def staged(evs, flush=None):
        # identical launches to lh_forward (+ lh_backward), with events between
        # stages; with `flush`, L2 is overwritten before each stage (evs: start,
        # end per stage)
        launches = [
            lambda: lh.lh_build_pyramid_score(shp, dt, q, k, v, pq, pk, pv, score, sp),
            lambda: lh.lh_topk_select(shp, score, idx, pos, slot, tws, tbw, sp),
            lambda: lh.lh_gather(shp, dt, q, k, v, pq, pk, pv, idx, qs, ks, vs, sp),
            lambda: lh.lh_subseq_attn_fwd(shp, qs, ks, vs, 0.0, os_, lse, sp),
            lambda: lh.lh_scatter_back(shp, dt, os_, slot, o, ic, sp),
        ]
        if backward:
            launches += [
                lambda: lh.lh_scatter_back_bwd(shp, dt, dO, slot, ic, dos, sp),
                lambda: lh.lh_subseq_attn_bwd(shp, qs, ks, vs, os_, lse, dos, 0.0, dqs, dks, dvs,
                                              aws, abw, sp),
                lambda: lh.lh_gather_bwd(shp, dt, dqs, dks, dvs, slot, dq, dk, dv, sp),
            ]
        for i, launch in enumerate(launches):
            if flush is not None:
                flush()
            evs[2 * i].record(stream)
            launch()
            evs[2 * i + 1].record(stream)

    def replay(flush=None, reps=steps):
        evs_all = []
        torch.cuda.synchronize()
        for _ in range(reps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(stages))]
            staged(evs, flush)
            evs_all.append(evs)
        torch.cuda.synchronize()
        return {st: statistics.mean(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs_all)
                for i, st in enumerate(stages)}

    with torch.cuda.stream(stream):
        stage_ms = replay()
        # the same launches with L2 overwritten (a 256 MB write, twice L2) before
        # each stage: no stage reads what the one before left in L2
        l2_junk = torch.empty(64 << 20, dtype=torch.float32, device=dev)
        stage_ms_flushed = replay(lambda: l2_junk.fill_(1.0), reps=max(3, min(steps, 10)))
        del l2_junk
        status |= lh.lh_read_device_status(stream)

    # rows the pooled gather must read: p^level for every selected entry
    gids = idx.view(U, w.S).long()
    offs = torch.tensor([sum(w.level_len(m) for m in range(l)) for l in range(w.L + 1)], device=dev)
    lev = torch.bucketize(gids, offs[1:], right=True)
    span_rows = int((torch.tensor(w.p, device=dev, dtype=torch.float64) ** lev).sum().item())
    alg = algorithmic(w, span_rows)
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    traffic_key = w.name if w.H == WORKLOADS.get(w.name, w).H else ""
    report = {}
    for st in stages:
        t = stage_ms[st] / 1e3
        if st.startswith("attn"):
            fl = alg[st + "_flop"]
            report[st] = {"ms": stage_ms[st], "tflops": fl / t / 1e12, "frac_tc": fl / t / 1e12 / tc}
        else:
            bts = alg[st]
            tf = stage_ms_flushed[st] / 1e3
            report[st] = {"ms": stage_ms[st], "gbs": bts / t / 1e9, "frac_hbm": bts / t / 1e9 / hbm,
                          "ms_l2_flushed": stage_ms_flushed[st],
                          "frac_hbm_l2_flushed": bts / tf / 1e9 / hbm}
        report[st]["traffic"] = measured_traffic(traffic_key, st)
    return {"ms_step": ms_step, "ms_fwd": ms_fwd, "stages": report, "status": status,
            "peak_bytes": peak_bytes, "clk": clk, "traffic_key": traffic_key,
            "tensors": {"x": x, "o": o, "dq": dq, "dk": dk, "dv": dv}, "shp": shp, "dt": dt,
            "stream": stream}


def roofline_of(report, peaks, peaks_src, traffic_key):
    """The roofline object of the stage that takes the longest."""
    dominant = max(report, key=lambda st: report[st]["ms"])
    r = report[dominant]
    if dominant.startswith("attn"):
        return {"kernel": dominant, "bound": "tensor", "achieved": r["tflops"],
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": r["frac_tc"],
                "traffic": measured_traffic(traffic_key, dominant),
                "peak_source": f"{peaks_src} bf16_tflops (burst)"}
    return {"kernel": dominant, "bound": "hbm", "achieved": r["gbs"], "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": r["frac_hbm"], "traffic": measured_traffic(traffic_key, dominant),
            "peak_source": f"{peaks_src} hbm_gbs"}


def extra_leg(lh, name, args, rk, dev, peaks, peaks_src, dense=False):
    """A further workload of the metric (the 512K and 1M contexts), measured the same
    way with a few steps; reported beside the main line, not as its value."""
    w = WORKLOADS[name]
    m = measure(lh, w, args, rk, dev, peaks, steps=5, warmup=3)
    tokens = w.B * w.N
    leg = {"config": workload_config(w, rk.world, "tcgen05"),
           "tokens_per_s": replicas.job_rate(tokens, rk.world, m["ms_step"] / 1e3),
           "fwd_tokens_per_s": replicas.job_rate(tokens, rk.world, m["ms_fwd"] / 1e3),
           "ms_per_step": m["ms_step"], "ms_fwd": m["ms_fwd"], "stages": m["stages"],
           "roofline": roofline_of(m["stages"], peaks, peaks_src, m["traffic_key"]),
           "peak_hbm_bytes": m["peak_bytes"], "device_status": m["status"]}
    if dense:
        t = m["tensors"]
        leg["dense_sdpa"] = dense_sdpa(w, t["x"]["q"], t["x"]["k"], t["x"]["v"], t["x"]["dO"],
                                       m["stream"], args, n=2)
        if "fwd_ms" in leg["dense_sdpa"]:
            leg["speedup_vs_dense"] = {"fwd": leg["dense_sdpa"]["fwd_ms"] / m["ms_fwd"],
                                       "fwd_bwd": leg["dense_sdpa"]["fwd_bwd_ms"] / m["ms_step"]}
    del m
    torch.cuda.empty_cache()
    return leg


def block_leg(w, args, dev, steps=5, warmup=3):
    """A causal self-attention block (fused Q/K/V projection, the layer, output
    projection; long_context_lh_b200.block) on the workload's shape, d_model = H*d:
    one training step = forward, backward of a mean-square loss and an SGD update,
    timed with CUDA events; beside it the same block with dense causal SDPA."""
    from long_context_lh_b200.block import DenseBlock, LighthouseBlock
    torch.manual_seed(0)
    dm = w.H * w.d
    x = torch.randn((w.B, w.N, dm), device=dev).to(torch.bfloat16)
    out = {"d_model": dm, "heads": w.H, "tokens": w.B * w.N}
    for name, cls in (("lighthouse", LighthouseBlock), ("dense", DenseBlock)):
        blk = cls(dm, w.H, w.p, w.L, w.S, device=dev)
        opt = torch.optim.SGD(blk.parameters(), lr=1e-3)

        def step():
            opt.zero_grad(set_to_none=True)
            y = blk(x)
            (y.float() ** 2).mean().backward()
            opt.step()

        n = steps if name == "lighthouse" else max(1, min(steps, 2))
        for _ in range(warmup if name == "lighthouse" else 1):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        out[name] = {"ms_per_step": ms, "tokens_per_s": w.B * w.N / (ms / 1e3)}
        del blk, opt
        torch.cuda.empty_cache()
    out["speedup_vs_dense"] = out["dense"]["ms_per_step"] / out["lighthouse"]["ms_per_step"]
    return out


def run_topk_compare(args, rk):
    """Both top-K implementations (one cluster per unit, device-wide passes) on the
    same scores at the pretraining and 512K-token shapes: CUDA-event medians and
    whether the selections are equal bit for bit; one JSON line."""
    from long_context_lh_b200 import lighthouse as lh
    from long_context_lh_b200.synth import WORKLOADS, make_inputs
    dev = torch.device("cuda", rk.local_rank)
    torch.cuda.set_device(dev)
    points = []
    for name in ("pretrain", "long"):
        w = WORKLOADS[name]
        x = make_inputs(w, dev, with_dO=False)
        shp = lh.make_shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)
        U, M = w.B * w.H, lh.lh_num_entries(shp)
        score = torch.empty(U * M, dtype=torch.float32, device=dev)
        lh.lh_score(shp, lh.dtype_code(x["q"].dtype), x["q"], x["k"], score)
        res, outs = {}, {}
        for impl in ("cluster", "passes"):
            idx = torch.empty(U * w.S, dtype=torch.int32, device=dev)
            pos = torch.empty_like(idx)
            slot = torch.empty(U * M, dtype=torch.int32, device=dev)
            wsb = lh.lh_topk_workspace_bytes(shp) if impl == "passes" else 0
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None
            run = lambda: lh.lh_topk_select(shp, score, idx, pos, slot, ws, wsb)  # noqa: E731
            for _ in range(args.warmup):
                run()
            ts = []
            for _ in range(max(args.steps, 5)):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                run()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            res[impl] = statistics.median(ts) * 1e3
            outs[impl] = (idx, pos, slot)
        equal = all(torch.equal(a, b) for a, b in zip(outs["cluster"], outs["passes"]))
        points.append({"workload": name, "entries_per_unit": M, "us_cluster": res["cluster"],
                       "us_passes": res["passes"], "equal": equal,
                       "lh_forward_uses": ["cluster", "passes"][lh.lh_forward_topk_path(shp)]})
        del x, score
        torch.cuda.empty_cache()
    if rk.rank == 0:
        print(json.dumps({"topk_compare": points, "device_status": lh.lh_read_device_status()}))


def run_sweep(args, rk):
    """Forward-only per-stage times over the hyperparameter sweep (p, L, S) at the
    pretraining shape; one JSON line."""
    from long_context_lh_b200 import lighthouse as lh
    from long_context_lh_b200.synth import sweep_workloads
    dev = torch.device("cuda", rk.local_rank)
    torch.cuda.set_device(dev)
    peaks, peaks_src = load_peaks()
    points = []
    for w in sweep_workloads():
        m = measure(lh, w, args, rk, dev, peaks, steps=max(1, min(args.steps, 10)),
                    warmup=args.warmup, backward=False)
        points.append({"p": w.p, "L": w.L, "S": w.S, "M": w.M, "ms_fwd": m["ms_fwd"],
                       "fwd_tokens_per_s": w.B * w.N / (m["ms_fwd"] / 1e3),
                       "stages_ms": {k: v["ms"] for k, v in m["stages"].items()},
                       "attn_fwd_frac_tc": m["stages"]["attn_fwd"]["frac_tc"]})
        del m
        torch.cuda.empty_cache()
    if rk.rank == 0:
        print(json.dumps({"metric": METRIC, "sweep": points, "n_gpus": 1, "peaks_source": peaks_src,
                          "config": {"workload": "sweep: B=1 H=16 N=98304 d=64 bf16, p x L x S"}}),
              flush=True)


def run_ours(args, rk):
    from long_context_lh_b200 import lighthouse as lh

    rank, world, local_rank = rk.rank, rk.world, rk.local_rank
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    if args.attn == "mma":
        lh.lh_set_attention_impl(1)
    elif args.attn == "tc":
        lh.lh_set_attention_impl(0)
    peaks, peaks_src = load_peaks()
    m = measure(lh, w, args, rk, dev, peaks, steps=args.steps, warmup=args.warmup,
                batch=rank, clocks=True)
    ms_step, ms_fwd, stage_report, status = m["ms_step"], m["ms_fwd"], m["stages"], m["status"]
    tokens = w.B * w.N
    value = replicas.job_rate(tokens, world, ms_step / 1e3)
    roof = roofline_of(stage_report, peaks, peaks_src, m["traffic_key"])
    t = m["tensors"]
    x = t["x"]

    # dense causal attention (torch SDPA, flash/cuDNN backend) on the same shapes
    dense = None
    if not args.no_dense and rank == 0:
        dense = dense_sdpa(w, x["q"], x["k"], x["v"], x["dO"], m["stream"], args)

    # end to end through the public API with pinned host buffers
    e2e = None if args.no_e2e else e2e_run(lh, w, m["shp"], m["dt"], x, dev, m["stream"], args, rk,
                                          {"o": t["o"], "dq": t["dq"], "dk": t["dk"], "dv": t["dv"]})
    launches = launches_per_step(lh, w)
    clk = m["clk"]
    del m, t, x
    torch.cuda.empty_cache()
    # the metric's other context lengths, on one GPU only (the scaling runs stay short)
    extra = {}
    if world == 1 and not args.heads and args.workload == "pretrain":
        for name in [n for n in args.also.split(",") if n]:
            extra[name] = extra_leg(lh, name, args, rk, dev, peaks, peaks_src,
                                    dense=(name == "long" and not args.no_dense))
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 io, fp16 MMA operands / fp32 accumulate",
        "data": "synthetic (seeded N(0,1) Q/K/V/dO, 1% tokens x4; no corpus or weights)",
        "config": workload_config(w, world,
                                  {0: "tcgen05", 1: "mma_sync", 2: "tcgen05 fwd, mma_sync bwd"}[
                                      lh.lh_attention_impl_in_use()]),
        "fwd_tokens_per_s": replicas.job_rate(tokens, world, ms_fwd / 1e3), "ms_fwd": ms_fwd,
        "roofline": roof, "stages": stage_report, "dense_sdpa": dense, "e2e": e2e,
        "gpu_launches": launches * args.steps, "gpu_launches_per_step": launches,
        "device_status": status, "peaks": peaks, "peaks_source": peaks_src,
    }
    if dense and "fwd_ms" in dense:
        out["speedup_vs_dense"] = {"fwd": dense["fwd_ms"] / ms_fwd, "fwd_bwd": dense["fwd_bwd_ms"] / ms_step}
    out.update(extra)
    if world == 1 and not args.heads and args.workload == "pretrain" and args.block:
        out["attention_block"] = block_leg(w, args, dev)
    if rank == 0:
        out["clocks"] = clk.summary()
        if not args.no_cpu:
            out["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
            # the same oracle on one core: one head, forward + backward
            one = cpu_baseline(w, steps=1, nthreads=1)
            out["cpu_baseline_1core"] = {k: one[k] for k in ("value", "unit", "cores", "kind", "sample")}
        print(json.dumps(out), flush=True)


def workload_config(w, world, attention):
    """The config object both arms print (same workload, same keys)."""
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} p={w.p} L={w.L} S={w.S} {w.dtype}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "p": w.p, "L": w.L, "S": w.S,
            "l2": "inputs larger than L2 (3 x %.0f MB + dO), no flush" % (w.B * w.H * w.N * w.d * 2 / 1e6),
            "attention": attention,
            "parallelism": f"replicas x{world} (heads independent)"}


def launches_per_step(lh, w):
    """Kernels of this library launched per step (lh_forward + lh_backward)."""
    shp = lh.make_shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S)
    dt = lh.dtype_code(w.torch_dtype)
    return lh.lh_kernel_launches(shp, dt, False) + lh.lh_kernel_launches(shp, dt, True)


def dense_sdpa(w, q, k, v, dO, stream, args, n=None):
    import torch.nn.functional as F
    try:
        qd = q.detach().requires_grad_(True)
        kd = k.detach().requires_grad_(True)
        vd = v.detach().requires_grad_(True)
        with torch.cuda.stream(stream):
            def f():
                return F.scaled_dot_product_attention(qd, kd, vd, is_causal=True)

            def fb():
                out = F.scaled_dot_product_attention(qd, kd, vd, is_causal=True)
                out.backward(dO)

            for _ in range(2):
                with torch.no_grad():
                    f()
                fb()
            torch.cuda.synchronize()
            n = max(1, min(args.steps, 5)) if n is None else n
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            for _ in range(n):
                with torch.no_grad():
                    f()
            e1.record(stream)
            for _ in range(n):
                fb()
            e2.record(stream)
            torch.cuda.synchronize()
        return {"fwd_ms": e0.elapsed_time(e1) / n, "fwd_bwd_ms": e1.elapsed_time(e2) / n,
                "backend": "torch.nn.functional.scaled_dot_product_attention(is_causal=True)"}
    except Exception as ex:  # pragma: no cover
        return {"error": str(ex)[:200]}


def e2e_run(lh, w, shp, dt, x, dev, stream, args, rk, ref_out):
    """The step through the public API (lh_forward, lh_backward) with the inputs
    copied up from pinned host memory and the results copied back inside the
    timed region.  Units (batch x head) are independent, so the step runs in C
    chunks of units pipelined over three streams: chunk i+1's inputs go up while
    chunk i computes and chunk i-1's results come down.  Same bytes and the same
    work per step as one whole-batch call; each chunk is an lh_forward +
    lh_backward on a shape with fewer heads."""
    U = w.B * w.H
    C = next(c for c in (8, 4, 2, 1) if U % c == 0)
    uc = U // C
    shp_c = lh.make_shape(1, uc, w.N, w.d, w.p, w.L, w.S)
    names_in, names_out = ("q", "k", "v", "dO"), ("o", "dq", "dk", "dv")
    host_in = {n: x[n].reshape(U, w.N, w.d).cpu().pin_memory() for n in names_in}
    host_out = {n: torch.empty((U, w.N, w.d), dtype=x["q"].dtype).pin_memory() for n in names_out}
    dbuf = [{n: torch.empty((uc, w.N, w.d), dtype=x["q"].dtype, device=dev)
             for n in names_in + names_out} for _ in range(2)]
    saved = torch.empty(lh.lh_saved_bytes(shp_c), dtype=torch.uint8, device=dev)
    wsb = lh.lh_workspace_bytes(shp_c, dt, True)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    s_in, s_comp, s_out = torch.cuda.Stream(device=dev), stream, torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    sp = s_comp.cuda_stream

    def step():
        for i in range(C):
            sl, b = slice(i * uc, (i + 1) * uc), dbuf[i & 1]
            s_in.wait_event(comp_done[i & 1])  # chunk i-2 has read these inputs
            with torch.cuda.stream(s_in):
                for n in names_in:
                    b[n].copy_(host_in[n][sl], non_blocking=True)
            in_done[i & 1].record(s_in)
            s_comp.wait_event(in_done[i & 1])
            s_comp.wait_event(out_done[i & 1])  # chunk i-2's results are down
            lh.lh_forward(shp_c, dt, b["q"], b["k"], b["v"], 0.0, b["o"], saved, ws, wsb, sp)
            lh.lh_backward(shp_c, dt, saved, b["dO"], 0.0, b["dq"], b["dk"], b["dv"], ws, wsb, sp)
            comp_done[i & 1].record(s_comp)
            s_out.wait_event(comp_done[i & 1])
            with torch.cuda.stream(s_out):
                for n in names_out:
                    host_out[n][sl].copy_(b[n], non_blocking=True)
            out_done[i & 1].record(s_out)

    K = max(1, min(args.steps, 10))
    step()
    torch.cuda.synchronize()
    replicas.barrier(rk)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(K):
        step()
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = replicas.max_over_ranks(rk, e0.elapsed_time(e1) / K, dev)
    # the chunked results must be the whole-batch results, bit for bit
    same = all(torch.equal(host_out[n].view(-1), ref_out[n].reshape(-1).cpu()) for n in names_out)
    return {"value": replicas.job_rate(w.B * w.N, rk.world, ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "chunks": C, "matches_device_run": same}


# ------------------------------------------------------------- CPU oracle
def oracle_step(w, h, x_np, nthreads=None):
    """Oracle forward + backward of head h (all of its tokens); nthreads: the
    oracle's worker threads (None: one per host core)."""
    import oracle
    s1 = oracle.Shape(1, 1, w.N, w.d, w.p, w.L, w.S)
    q, k, v, dO = (x_np[n][:, h:h + 1] for n in ("q", "k", "v", "dO"))
    f = oracle.forward(s1, q, k, v, nthreads=nthreads)
    oracle.backward(s1, f, dO, nthreads=nthreads)


def cpu_baseline(w, budget_s=20.0, steps=None, warmup=0, nthreads=None):
    """Time the oracle on this host's cores (or on `nthreads` of them): whole
    heads, until the budget is spent."""
    import numpy as np  # noqa: F401
    xc = make_inputs(w, "cpu")
    x_np = {n: t.float().numpy() for n, t in xc.items()}
    cores = nthreads or os.cpu_count() or 1
    for h in range(warmup):
        oracle_step(w, h % w.H, x_np, nthreads)
    t0 = time.perf_counter()
    heads = 0
    times = []
    while heads < w.H:
        t1 = time.perf_counter()
        oracle_step(w, heads % w.H, x_np, nthreads)
        times.append(time.perf_counter() - t1)
        heads += 1
        if steps is not None and heads >= steps:
            break
        if steps is None and time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    value = w.B * w.N * (heads / w.H) / el
    return {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {w.H} heads of the {w.name} workload, forward+backward, "
                      f"{el:.1f} s; tokens/s = B*N*(heads/H)/time",
            "per_head_s": times}


def run_reference(args, rk):
    if rk.rank != 0:  # the CPU oracle runs once, on rank 0; the other ranks exit
        return
    world = rk.world
    w = WORKLOADS[args.workload]
    cb = cpu_baseline(w, steps=args.steps, warmup=args.warmup)
    out = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": 1e3 * sum(cb["per_head_s"]) / max(len(cb["per_head_s"]), 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1) Q/K/V/dO, 1% tokens x4; no corpus or weights)",
           "config": workload_config(w, world, "CPU oracle (fp64), one head per step"),
           "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
           "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="pretrain", choices=["pretrain", "long", "extreme"])
    ap.add_argument("--attn", default="auto", choices=["auto", "tc", "mma"])
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (smaller cases for profiler captures; not a bench line)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--also", default="long,extreme",
                    help="further workloads measured beside the main line (1 GPU; '' for none)")
    ap.add_argument("--block", type=int, default=1,
                    help="1: also time a training step of the attention block (1 GPU)")
    ap.add_argument("--sweep", action="store_true",
                    help="forward-only per-stage times over the p x L x S sweep (one JSON line)")
    ap.add_argument("--topk-compare", action="store_true",
                    help="both top-K implementations at the pretraining and 512K shapes (one JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    rk = replicas.from_env()
    if args.impl == "reference":
        run_reference(args, rk)
        return
    if rk.multi:
        torch.cuda.set_device(rk.local_rank)
    replicas.init(rk, "nccl", 300.0, torch.device("cuda", rk.local_rank) if rk.multi else None)
    try:
        if args.sweep:
            run_sweep(args, rk)
        elif args.topk_compare:
            run_topk_compare(args, rk)
        else:
            run_ours(args, rk)
    finally:
        replicas.finish(rk)


if __name__ == "__main__":
    main()
