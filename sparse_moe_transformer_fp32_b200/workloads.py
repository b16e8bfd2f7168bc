"""Seeded synthetic inputs for the Beam sparse-MoE layer workloads.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no routing, no matmul, no normalisation).  The CUDA path,
its tests, the benchmark and the CPU oracle all take their inputs from here,
so that both sides of every parity check read the same bytes.

Shapes follow the Beam model card (Transformers ``beam.md``, "BeamConfig":
hidden_size 5120, moe_intermediate_size 2560, num_experts 256,
num_experts_per_tok 8, n_group 8, topk_group 4, routed_scaling_factor 2.5,
rms_norm_eps 1e-6).  The five workloads are:

* ``tiny``    T=64,    d=256,  E=16 in 4 groups, topk_group 2, top_k 4, I=128
* ``decode``  T=32,    Beam shapes
* ``prefill`` T=4096,  Beam shapes, near-uniform expert load
* ``skewed``  T=16384, Beam shapes, bias 0.5/rank over a seeded permutation
* ``block``   T=8192,  Beam shapes, FP32 residual input with sandwich norms
* ``dense``   T=4096,  dense SwiGLU MLP of the first layers (d=5120, intermediate 20480)

Distributions: hidden ~N(0,1) rounded to BF16; router weight FP32 normal with
the stated standard deviation; expert weights BF16 normal with variance
1/fan_in (gate/up: 1/d, down: 1/I); bias FP32 uniform, or 0.5/rank for the
skewed workload; norm gains ~U(0.9, 1.1); residual x ~N(0,1) FP32.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = [
    "Workload", "WORKLOADS", "seed_for", "router_weight", "router_bias",
    "hidden", "hidden_row", "residual_x", "residual_row", "norm_gains",
    "expert_weight", "expert_weights",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    n_group: int
    topk_group: int
    top_k: int
    I: int
    seed: int
    router_std: float
    bias_kind: str            # "uniform" or "inv_rank"
    bias_range: float         # half-width for "uniform", numerator for "inv_rank"
    scale: float = 2.5        # routed_scaling_factor
    norm_topk_prob: bool = True
    block: bool = False       # sandwich RMSNorms + depth-scaled residual around the layer
    dense: bool = False       # dense SwiGLU MLP (one "expert", no routing)
    eps: float = 1e-6
    k_resid: int = 10

    @property
    def R(self) -> int:
        """(token, expert) slots: T * top_k."""
        return self.T * self.top_k

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)


_BEAM = dict(d=5120, E=256, n_group=8, topk_group=4, top_k=8, I=2560, router_std=0.01)

WORKLOADS = {
    "tiny": Workload("tiny", T=64, d=256, E=16, n_group=4, topk_group=2, top_k=4, I=128,
                     seed=0, router_std=0.02, bias_kind="uniform", bias_range=0.1),
    "decode": Workload("decode", T=32, seed=1, bias_kind="uniform", bias_range=0.05, **_BEAM),
    "prefill": Workload("prefill", T=4096, seed=2, bias_kind="uniform", bias_range=0.05, **_BEAM),
    "skewed": Workload("skewed", T=16384, seed=3, bias_kind="inv_rank", bias_range=0.5, **_BEAM),
    "block": Workload("block", T=8192, seed=4, bias_kind="uniform", bias_range=0.05, block=True,
                      **_BEAM),
    # Beam's first three layers: dense SwiGLU MLP, intermediate_size 20480
    "dense": Workload("dense", T=4096, d=5120, E=1, n_group=1, topk_group=1, top_k=1, I=20480,
                      seed=5, router_std=0.0, bias_kind="uniform", bias_range=0.0, dense=True),
}

# tensor ids for seed derivation
_ID = {"router": 1, "bias": 2, "hidden": 3, "hidden_row": 4, "gate": 5, "up": 6, "down": 7,
       "x": 8, "x_row": 9, "g_pre": 10, "g_post": 11}


def seed_for(*parts: int) -> int:
    """Mixes integers into one 63-bit generator seed (splitmix64 finaliser per part)."""
    z = 0x9E3779B97F4A7C15
    mask = (1 << 64) - 1
    for p in parts:
        z = (z + (int(p) & mask) + 0x9E3779B97F4A7C15) & mask
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
        z ^= z >> 31
    return z & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(*parts))
    return g


def router_weight(w: Workload, device="cpu") -> torch.Tensor:
    """FP32 [E, d], normal with standard deviation ``router_std``."""
    g = _gen(device, w.seed, _ID["router"])
    return torch.randn(w.E, w.d, generator=g, device=device, dtype=torch.float32) * w.router_std


def router_bias(w: Workload, device="cpu") -> torch.Tensor:
    """FP32 [E].  uniform(-r, r), or 0.5/rank(e) with rank 1 + position of e in a
    seeded random permutation (so a handful of hot experts take most tokens)."""
    g = _gen("cpu", w.seed, _ID["bias"])
    if w.bias_kind == "uniform":
        b = (torch.rand(w.E, generator=g, dtype=torch.float64) * 2.0 - 1.0) * w.bias_range
    elif w.bias_kind == "inv_rank":
        perm = torch.randperm(w.E, generator=g)
        rank = torch.empty(w.E, dtype=torch.float64)
        rank[perm] = torch.arange(1, w.E + 1, dtype=torch.float64)
        b = w.bias_range / rank
    else:
        raise ValueError(w.bias_kind)
    return b.to(torch.float32).to(device)


def hidden(w: Workload, device="cpu") -> torch.Tensor:
    """BF16 [T, d] ~N(0,1)."""
    g = _gen("cpu", w.seed, _ID["hidden"])
    return torch.randn(w.T, w.d, generator=g, dtype=torch.float32).to(torch.bfloat16).to(device)


def hidden_row(w: Workload, t: int, attempt: int) -> torch.Tensor:
    """A fresh BF16 [d] draw for token ``t``, the ``attempt``-th replacement."""
    g = _gen("cpu", w.seed, _ID["hidden_row"], t, attempt)
    return torch.randn(w.d, generator=g, dtype=torch.float32).to(torch.bfloat16)


def residual_x(w: Workload, device="cpu") -> torch.Tensor:
    """FP32 [T, d] residual stream ~N(0,1) for the block workload."""
    g = _gen("cpu", w.seed, _ID["x"])
    return torch.randn(w.T, w.d, generator=g, dtype=torch.float32).to(device)


def residual_row(w: Workload, t: int, attempt: int) -> torch.Tensor:
    g = _gen("cpu", w.seed, _ID["x_row"], t, attempt)
    return torch.randn(w.d, generator=g, dtype=torch.float32)


def norm_gains(w: Workload, device="cpu"):
    """(g_pre, g_post), FP32 [d] each, ~U(0.9, 1.1)."""
    out = []
    for name in ("g_pre", "g_post"):
        g = _gen("cpu", w.seed, _ID[name])
        out.append((0.9 + 0.2 * torch.rand(w.d, generator=g, dtype=torch.float64))
                   .to(torch.float32).to(device))
    return tuple(out)


def expert_weight(w: Workload, which: str, e: int, device="cpu") -> torch.Tensor:
    """One expert's BF16 matrix in nn.Linear layout (out x in):
    gate/up [I, d] with std 1/sqrt(d); down [d, I] with std 1/sqrt(I)."""
    if which in ("gate", "up"):
        shape, fan_in = (w.I, w.d), w.d
    elif which == "down":
        shape, fan_in = (w.d, w.I), w.I
    else:
        raise ValueError(which)
    g = _gen(device, w.seed, _ID[which], e)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (x * (1.0 / math.sqrt(fan_in))).to(torch.bfloat16)


def expert_weights(w: Workload, device="cpu"):
    """(w_gate [E,I,d], w_up [E,I,d], w_down [E,d,I]) BF16, drawn expert by expert on ``device``."""
    wg = torch.empty(w.E, w.I, w.d, dtype=torch.bfloat16, device=device)
    wu = torch.empty_like(wg)
    wd = torch.empty(w.E, w.d, w.I, dtype=torch.bfloat16, device=device)
    for e in range(w.E):
        wg[e] = expert_weight(w, "gate", e, device)
        wu[e] = expert_weight(w, "up", e, device)
        wd[e] = expert_weight(w, "down", e, device)
    return wg, wu, wd
