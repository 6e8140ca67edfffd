"""Seeded synthetic workloads shaped like the pages' models.

This module holds no quantization, routing-grouping or forward arithmetic: it only
draws inputs.  Both the CUDA path (tests, bench) and the CPU oracle (tests) are fed
from here.  The checkpoints the pages measure on (OLMoE-1B-7B, Qwen3-30B-A3B,
Mixtral-8x7B) are not available, so seeded tensors of the same shapes stand in:

* expert weights: fp32 N(0, 0.02) drawn with ``torch.Generator(seed)``, rounded
  once to bf16 (int8 workload: an iid Bernoulli(0.001) outlier mask multiplies the
  masked fp32 values by 20 before that rounding);
* hidden states: bf16 N(0, 1);
* routing: fp32 N(0, 1) logits ``[T, E]`` (plus a Zipf(1.2) per-expert bias for the
  skewed workload), softmax over E, top-K with ties to the lower expert id, the K
  weights renormalised to sum to 1 (fp32).

Seeds: ``seed = 1000 * cfg + {0: gate_up, 1: down, 2: hidden, 3: logits,
4: gate_up outlier mask, 5: Zipf permutation, 6: down outlier mask}``.
"""
from __future__ import annotations

import dataclasses
import math

import torch

MODE_NF4, MODE_NF4_DQ, MODE_INT8 = 0, 1, 2
MODE_NAMES = {MODE_NF4: "nf4", MODE_NF4_DQ: "nf4_dq", MODE_INT8: "int8"}


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    E: int
    H: int
    I: int
    K: int
    T: int
    mode: int
    outliers: bool = False
    zipf: float = 0.0
    layers: int = 1          # layers quantized on load (Qwen-like: 48)

    @property
    def label(self) -> str:
        return (f"{self.name}: E={self.E} H={self.H} I={self.I} top-{self.K} "
                f"T={self.T} {MODE_NAMES[self.mode]}")


WORKLOADS = {
    "tiny": Workload(1, "tiny", 8, 256, 128, 2, 64, MODE_NF4),
    "olmoe": Workload(2, "olmoe", 64, 2048, 1024, 8, 4096, MODE_NF4),
    "qwen": Workload(3, "qwen", 128, 2048, 768, 8, 8192, MODE_NF4_DQ, layers=48),
    "mixtral": Workload(4, "mixtral", 8, 4096, 14336, 2, 16384, MODE_INT8, outliers=True),
    "skew1": Workload(5, "skew1", 128, 2048, 768, 8, 1, MODE_NF4, zipf=1.2),
    "skew64": Workload(5, "skew64", 128, 2048, 768, 8, 64, MODE_NF4, zipf=1.2),
    "skew32k": Workload(5, "skew32k", 128, 2048, 768, 8, 32768, MODE_NF4, zipf=1.2),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def expert_weights(E: int, R: int, C: int, seed: int, outliers: bool = False,
                   device="cpu", out: torch.Tensor | None = None,
                   mask_seed: int | None = None) -> torch.Tensor:
    """bf16 ``[E, R, C]`` from fp32 N(0, 0.02) rounded once (optional x20 outliers).

    Drawn one expert at a time so that large tensors need one expert of fp32
    scratch.  ``out`` (bf16, same shape) is filled in place when given.
    """
    g = _gen(seed, device)
    gm = _gen(seed + 4 if mask_seed is None else mask_seed, device) if outliers else None
    if out is None:
        out = torch.empty((E, R, C), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w = torch.randn((R, C), generator=g, dtype=torch.float32, device=device) * 0.02
        if outliers:
            m = torch.rand((R, C), generator=gm, dtype=torch.float32, device=device) < 0.001
            w = torch.where(m, w * 20.0, w)
        out[e].copy_(w.to(torch.bfloat16))
    return out


def hidden_states(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn((T, H), generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def routing(T: int, E: int, K: int, seed: int, zipf: float = 0.0, device="cpu"):
    """(top_k_index int32 [T,K], top_k_weights fp32 [T,K]) from softmax-top-k."""
    g = _gen(seed, device)
    logits = torch.randn((T, E), generator=g, dtype=torch.float32, device=device)
    if zipf:
        gp = _gen(seed + 2, "cpu")   # seed + 2 == 1000*cfg + 5 (Zipf permutation)
        r = torch.randperm(E, generator=gp).to(torch.float64) + 1.0
        bias = (-zipf * torch.log(r)).to(torch.float32).to(device)
        logits = logits + bias
    p = torch.softmax(logits, dim=-1)
    order = torch.argsort(-p, dim=-1, stable=True)[:, :K]
    w = torch.gather(p, 1, order)
    w = w / w.sum(dim=-1, keepdim=True)
    return order.to(torch.int32), w.contiguous()


def workload_inputs(wl: Workload, device="cpu", T: int | None = None):
    """All inputs of one layer of a workload: dict of torch tensors."""
    T = wl.T if T is None else T
    s = 1000 * wl.cfg
    gu = expert_weights(wl.E, 2 * wl.I, wl.H, s + 0, wl.outliers, device)
    dn = expert_weights(wl.E, wl.H, wl.I, s + 1, wl.outliers, device, mask_seed=s + 6)
    x = hidden_states(T, wl.H, s + 2, device)
    idx, w = routing(T, wl.E, wl.K, s + 3, wl.zipf, device)
    return {"gate_up": gu, "down": dn, "hidden": x, "top_k_index": idx, "top_k_weights": w}


def forward_flops(T: int, K: int, H: int, I: int) -> float:
    """Algorithmic FLOPs of the routed experts forward: 2*T*K*(2I*H + H*I)."""
    return 6.0 * T * K * H * I


def quantize_bytes(mode: int, E: int, R: int, C: int) -> float:
    """Algorithmic HBM bytes of quantizing one [E,R,C] bf16 tensor: read + write."""
    n = E * R * C
    if mode == MODE_NF4:
        return 2.0 * n + n / 2 + 4.0 * n / 64
    if mode == MODE_NF4_DQ:
        nb = n // 64
        return 2.0 * n + n / 2 + nb + 4.0 * math.ceil(R * C / 64 / 256) * E + 4.0 * E
    return 3.0 * n + 4.0 * E * R
