"""Seeded synthetic inputs for the dropless top-k MoE layer.

This module only draws random numbers and lays them out. It holds none of the
layer's arithmetic (no routing, no softmax, no FFN), so both the CUDA path and
the CPU oracle may take their inputs from it.

Workloads (shapes from the OLMoE description in "Transformers 中的 OLMoE"
(blog.gitcode.com), section "OlmoeConfig" table, and from the expert-count /
fine-grained scaling study in the Olmo-core 3 news article (xxqk.cn),
section "关键数字"):

  tiny_fp32          T=256   d=128  E=8   k=2 F=256   fp32, logits from x·Wrᵀ
  olmoe_1b7b         T=16384 d=2048 E=64  k=8 F=1024  bf16, logits from x·Wrᵀ
  sweep_e{8,32,128}  T=8192  d=4096 k=4  F=2048       bf16, logits ~ N(0,1)
  sweep_e*_zipf      as above, logits ~ N(0,1) + ln p_e, p_e ∝ (e+1)^-1.1
  fine_grained_e384  T=4096  d=7168 E=384 k=8 F=2048  bf16, logits ~ N(0,1),
                     forward + backward
  mxfp8_e128         sweep_e128 with MXFP8 operands

Value recipe: x ~ N(0,1); router and expert weights ~ N(0, 0.02); every
value is rounded once to the layer dtype at generation, so every consumer
reads identical bytes. The upstream gradient dOut ~ N(0,1) uses seed+1.
Random numbers come from torch's seeded generator on the requested device;
the same seed on a different device type gives a different (but again
deterministic) draw, so a test always generates once and copies.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    F: int
    dtype: str = "bf16"          # "bf16" or "f32": layer (storage) dtype
    logits: str = "router"       # "router" (x·Wrᵀ), "normal", "zipf"
    mxfp8: bool = False
    backward: bool = False
    seed: int = 0
    zipf_s: float = 1.1
    weight_std: float = 0.02

    @property
    def R(self) -> int:
        return self.T * self.k

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> None:
    WORKLOADS[w.name] = w


_add(Workload("tiny_fp32", T=256, d=128, E=8, k=2, F=256, dtype="f32", logits="router"))
_add(Workload("olmoe_1b7b", T=16384, d=2048, E=64, k=8, F=1024, logits="router"))
for _E in (8, 32, 128):
    _add(Workload(f"sweep_e{_E}", T=8192, d=4096, E=_E, k=4, F=2048, logits="normal"))
    _add(Workload(f"sweep_e{_E}_zipf", T=8192, d=4096, E=_E, k=4, F=2048, logits="zipf"))
_add(Workload("fine_grained_e384", T=4096, d=7168, E=384, k=8, F=2048, logits="normal",
              backward=True))
_add(Workload("mxfp8_e128", T=8192, d=4096, E=128, k=4, F=2048, logits="normal", mxfp8=True))


def _gen(device: torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, std: float, g: torch.Generator, device, dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_log_popularity(E: int, s: float) -> torch.Tensor:
    """ln p_e with p_e ∝ (e+1)^-s, normalised (input construction only)."""
    e = torch.arange(1, E + 1, dtype=torch.float64)
    w = e.pow(-s)
    return (w / w.sum()).log()


def make_inputs(w: Workload, device="cpu", *, weights: bool = True,
                seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw every input of workload ``w`` on ``device``.

    Returns x [T,d]; Wr [E,d] (router workloads) or logits [T,E] fp32;
    W1, W3 [E,F,d] and W2 [E,d,F] (if ``weights``); dOut [T,d] for backward
    workloads. Expert weights are drawn one expert at a time so that the
    34 GB fine-grained workload never needs an fp32 staging copy of the
    whole tensor.
    """
    device = torch.device(device)
    seed = w.seed if seed is None else seed
    g = _gen(device, seed)
    dt = w.torch_dtype
    out: Dict[str, torch.Tensor] = {}
    out["x"] = _randn((w.T, w.d), 1.0, g, device, dt)
    if w.logits == "router":
        out["Wr"] = _randn((w.E, w.d), w.weight_std, g, device, dt)
    else:
        lg = torch.randn((w.T, w.E), generator=g, device=device, dtype=torch.float32)
        if w.logits == "zipf":
            lg += zipf_log_popularity(w.E, w.zipf_s).to(torch.float32).to(device)
        out["logits"] = lg
    if weights:
        W1 = torch.empty((w.E, w.F, w.d), dtype=dt, device=device)
        W3 = torch.empty((w.E, w.F, w.d), dtype=dt, device=device)
        W2 = torch.empty((w.E, w.d, w.F), dtype=dt, device=device)
        for e in range(w.E):
            W1[e] = _randn((w.F, w.d), w.weight_std, g, device, dt)
            W3[e] = _randn((w.F, w.d), w.weight_std, g, device, dt)
            W2[e] = _randn((w.d, w.F), w.weight_std, g, device, dt)
        out["W1"], out["W3"], out["W2"] = W1, W3, W2
    if w.backward:
        g2 = _gen(device, seed + 1)
        out["dOut"] = _randn((w.T, w.d), 1.0, g2, device, dt)
    return out


def adversarial_logits(T: int, E: int, kind: str, seed: int = 0) -> torch.Tensor:
    """Logits with ties and degenerate rows, for routing edge cases.

    kinds: "constant" (every row equal), "dups" (values drawn from a tiny
    set, so many exact ties), "signed_zero" (mix of +0.0 and -0.0 and a few
    ±1), "normal".
    """
    g = _gen(torch.device("cpu"), seed)
    if kind == "constant":
        return torch.full((T, E), 0.25, dtype=torch.float32)
    if kind == "dups":
        v = torch.randint(0, 3, (T, E), generator=g).to(torch.float32) * 0.5
        return v
    if kind == "signed_zero":
        s = torch.randint(0, 4, (T, E), generator=g)
        v = torch.zeros((T, E), dtype=torch.float32)
        v[s == 1] = -0.0
        v[s == 2] = 1.0
        v[s == 3] = -1.0
        return v
    if kind == "normal":
        return torch.randn((T, E), generator=g, dtype=torch.float32)
    raise ValueError(kind)


def bytes_of(w: Workload) -> Dict[str, int]:
    s = w.esize
    return {
        "x": w.T * w.d * s,
        "Xe": w.R * w.d * s,
        "H": w.R * w.F * s,
        "weights": 3 * w.E * w.d * w.F * s,
        "logits": w.T * w.E * 4,
    }


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "make_inputs", "adversarial_logits",
           "zipf_log_popularity", "bytes_of", "ceil_div"]
