"""Seeded synthetic inputs for the MoE layer (route -> dispatch -> expert MLP -> combine).

This module is shared by the tests, the CPU oracle's callers and ``bench.py``.
It holds the workload shapes and random-number recipes only: no step of the
layer's arithmetic lives here.

Workloads (shapes from the pages' settings, synthetic values):

* ``tiny``    fp32, T=64, H=128, E=8, K=2, F=256, S=2, cf=1.25
* ``mixtral`` bf16, T=4096, H=4096, E=8, K=2, F=14336, S=8, cf=1.25
  (Mixtral 8x7B is the model named in the pplx-kernels page, "Introductie")
* ``dsv3``    bf16 decode batch, T=1024, H=7168, E=256, K=8, F=2048, S=8, cf=1.5
  (hidden 7168 as in "Enabling trillion-parameter models on AWS EFA", "Оценка")
* ``skewed``  bf16, T=16384, H=2048, E=64, K=6, F=1408, S=8, cf=1.0,
  Zipf-skewed router (the "cross-rank skewed" routing mode of the
  "MoE Expert Parallel Benchmark" page, Step 1)
* ``kimi``    bf16 prefill, T=32768, H=7168, E=384, K=8, F=2048, S=16, cf=1.25
* ``kimi_seg`` one owner segment of ``kimi``: T=2048, E=24, S=1, the same
  rows per expert and capacity (a profiling case of a few GB)

Value recipe (all from one ``torch.Generator`` seeded with ``seed``, drawn in
this order): router logits N(0,1) [T,E] fp32; per-expert logit bias (dsv3:
N(0, 0.1) with 0.1 the standard deviation; skewed: 2*ln(rank^-1.2) with rank
e+1; others none) added to every token's logits; activations x N(0,1) [T,H];
gate/up weights N(0, 0.02^2) [E',2F,H] (rows 0..F-1 gate, F..2F-1 up); down
weights N(0, 0.02^2) [E',H,F], with E' = E + n_shared (a shared expert, when
present, is the last one).  Activations and weights are produced in the
workload's activation dtype.

``with_(n_shared=1)`` adds one shared expert of the routed experts' width, as
in DeepSeek-V3 and Kimi-K2 (one shared expert of width 2048 next to the routed
ones).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    K: int
    F: int
    S: int
    cf: float
    act: str              # "f32" or "bf16"
    bias: str = "none"    # "none" | "normal0.1" | "zipf1.2"
    row_align: int = 128  # A: expert start alignment inside the dispatch buffer
    n_shared: int = 0     # 1: one shared expert every token uses with weight 1

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_act(self) -> torch.dtype:
        return torch.float32 if self.act == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny": Workload("tiny", 64, 128, 8, 2, 256, 2, 1.25, "f32", row_align=1),
    "mixtral": Workload("mixtral", 4096, 4096, 8, 2, 14336, 8, 1.25, "bf16"),
    "dsv3": Workload("dsv3", 1024, 7168, 256, 8, 2048, 8, 1.5, "bf16", bias="normal0.1"),
    "skewed": Workload("skewed", 16384, 2048, 64, 6, 1408, 8, 1.0, "bf16", bias="zipf1.2"),
    "kimi": Workload("kimi", 32768, 7168, 384, 8, 2048, 16, 1.25, "bf16"),
    # one owner segment of the Kimi-K2 shape (24 experts) with the same rows
    # per expert (T*K/E = 683) and capacity (854): the case the profiler
    # captures, 2.1 GB of weights instead of 33.8 GB
    "kimi_seg": Workload("kimi_seg", 2048, 7168, 24, 8, 2048, 1, 1.25, "bf16"),
}


def logit_bias(w: Workload, gen: torch.Generator, device) -> torch.Tensor | None:
    """Per-expert additive logit bias of the synthetic router (fp32 [E]) or None."""
    if w.bias == "none":
        return None
    if w.bias == "normal0.1":
        return torch.randn(w.E, generator=gen, device=device, dtype=torch.float32) * 0.1
    if w.bias == "zipf1.2":
        ranks = torch.arange(1, w.E + 1, device=device, dtype=torch.float64)
        return (2.0 * torch.log(ranks ** -1.2)).to(torch.float32)
    raise ValueError(f"unknown bias kind {w.bias!r}")


def make_router_logits(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    logits = torch.randn(w.T, w.E, generator=gen, device=device, dtype=torch.float32)
    b = logit_bias(w, gen, device)
    if b is not None:
        logits += b[None, :]
    return logits


def _normal(shape, std, dtype, gen, device, chunk_elems=1 << 28):
    """N(0, std^2) in ``dtype``; drawn in fp32 chunks so that huge bf16 tensors
    never need a full fp32 copy."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        tmp = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[s:e].copy_(tmp)
    return out


def make_inputs(w: Workload, seed: int = 0, device="cpu", weights: bool = True,
                router: bool = False):
    """Return dict(logits, x, w_gu, w_d) drawn in a fixed order from one seeded
    generator; with router=True also the router weights w_g [E,H] ~ N(0, 1/H)
    (so that x w_g^T has unit variance) and a selection-only bias sel_bias [E]
    ~ N(0, 0.1^2), drawn after the others."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    logits = make_router_logits(w, gen, device)
    x = _normal((w.T, w.H), 1.0, w.torch_act, gen, device)
    out = {"logits": logits, "x": x}
    if weights:
        ew = w.E + w.n_shared
        out["w_gu"] = _normal((ew, 2 * w.F, w.H), 0.02, w.torch_act, gen, device)
        out["w_d"] = _normal((ew, w.H, w.F), 0.02, w.torch_act, gen, device)
    if router:
        out["w_g"] = _normal((w.E, w.H), w.H ** -0.5, w.torch_act, gen, device)
        out["sel_bias"] = torch.randn(w.E, generator=gen, device=device, dtype=torch.float32) * 0.1
    return out


def small_case(T, H, E, K, F, S, cf, act="bf16", row_align=128, bias="none",
               n_shared=0) -> Workload:
    """An ad-hoc workload for parity sweeps (ragged sizes, edge cases)."""
    name = f"case_T{T}_H{H}_E{E}_K{K}_F{F}" + ("_shared" if n_shared else "")
    return Workload(name, T, H, E, K, F, S, cf, act, bias, row_align, n_shared)


def tied_logits(T: int, E: int, levels: int, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """Router logits drawn from only ``levels`` distinct values, so that many
    ties occur (tie-break edge case)."""
    v = torch.randint(0, levels, (T, E), generator=gen, device=device)
    return (v.to(torch.float32) - levels / 2) * 0.5


def expected_bytes_gb(w: Workload) -> float:
    """Device memory held by the inputs, in GB (for sizing decisions)."""
    s = 4 if w.act == "f32" else 2
    return (w.T * w.E * 4 + w.T * w.H * s + 3 * (w.E + w.n_shared) * w.F * w.H * s) / 1e9


__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_router_logits", "small_case",
           "tied_logits", "expected_bytes_gb", "logit_bias"]
