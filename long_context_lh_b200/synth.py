"""Seeded synthetic inputs for one Lighthouse Attention layer.

This module holds the workload shapes and the random input recipe, and none of
the method's arithmetic: it only draws Q, K, V and dO.  Both the CUDA path and
the CPU oracle consume the same bytes (drawn once, then copied), so neither side
can disagree with the other because of its own random-number or libm code.

The pages train a 530M Llama-3-style decoder on C4 at 98,304 tokens of context
(gist.science/es "Resumen Técnico…", §4 Resultados Experimentales).  Neither the
corpus nor the weights are available here, so projected Q/K/V are drawn from the
distributions below, with the per-head shapes of that kind of model.

Recipe (torch.Generator, seeded; fp32 draws rounded to the tensor dtype):
  * "normal":    i.i.d. N(0, 1).
  * "outliers":  N(0, 1), then 1% of token positions (one seeded set per batch
                 row, shared by every head and by Q, K and V) scaled by 4, the
                 high-norm tokens a norm scorer is meant to find.
  * "lognormal": each token row is z * exp(0.5 g), z ~ N(0, 1)^d and one
                 g ~ N(0, 1) per (batch row, token), shared by heads and Q/K/V,
                 so per-token norms spread log-normally.
  dO is always i.i.d. N(0, 1).
Seeds: Q=1, K=2, V=3, dO=4, outlier mask=5, log-normal factors=6, each XORed
with 0x1F1F * workload id.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    B: int
    H: int
    N: int
    d: int
    p: int
    L: int
    S: int
    dtype: str  # "bf16" or "f32"
    dist: str  # "normal" | "outliers" | "lognormal"
    backward: bool

    def level_len(self, l: int) -> int:
        return self.N // self.p ** l

    @property
    def M(self) -> int:
        return sum(self.level_len(l) for l in range(self.L))

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # small case the CPU oracle finishes in seconds (fp32 inputs, forward only)
    "tiny": Workload("tiny", 1, 1, 2, 4096, 64, 4, 3, 512, "f32", "normal", False),
    # pretraining shape: the 98,304-token context of the pages' 530M model
    "pretrain": Workload("pretrain", 2, 1, 16, 98304, 64, 4, 4, 8192, "bf16", "outliers", True),
    # long context, 512K tokens
    "long": Workload("long", 4, 1, 16, 524288, 64, 4, 5, 16384, "bf16", "normal", True),
    # one-GPU extreme context, 1M tokens, d = 128
    "extreme": Workload("extreme", 5, 1, 8, 1048576, 128, 4, 6, 16384, "bf16", "lognormal", True),
}


def sweep_workloads():
    """Hyperparameter sweep at N=98,304, H=16, d=64 (forward only)."""
    base = WORKLOADS["pretrain"]
    out = []
    for p in (2, 4, 8):
        for L in (2, 3, 4, 5):
            for S in (4096, 8192, 16384):
                out.append(base.with_(name=f"sweep_p{p}_L{L}_S{S}", wid=3, p=p, L=L, S=S,
                                      dist="normal", backward=False))
    return out


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(w: Workload, device="cpu", with_dO: bool = True, batch: int = 0):
    """Draw q, k, v (and dO) of shape [B, H, N, d] in the workload's dtype.

    batch selects an independent draw of the same workload (the replica a rank
    of a multi-GPU run processes); batch 0 is the draw every test uses."""
    device = torch.device(device)
    salt = 0x1F1F * w.wid + 0x9E3779B1 * batch
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    scale_tok = None
    if w.dist == "outliers":
        scale_tok = torch.ones((w.B, 1, w.N, 1), dtype=torch.float32, device=device)
        g = _gen(device, 5 ^ salt)
        n_out = max(1, w.N // 100)
        for b in range(w.B):
            sel = torch.randperm(w.N, generator=g, device=device)[:n_out]
            scale_tok[b, 0, sel, 0] = 4.0
    elif w.dist == "lognormal":
        g = _gen(device, 6 ^ salt)
        gz = torch.randn((w.B, 1, w.N, 1), generator=g, device=device, dtype=torch.float32)
        scale_tok = torch.exp(0.5 * gz)
    for name, seed in (("q", 1), ("k", 2), ("v", 3)):
        g = _gen(device, seed ^ salt)
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if scale_tok is not None:
            x.mul_(scale_tok)
        out[name] = x.to(w.torch_dtype)
        del x
    if with_dO:
        g = _gen(device, 4 ^ salt)
        out["dO"] = torch.randn(shape, generator=g, device=device,
                                dtype=torch.float32).to(w.torch_dtype)
    return out
