"""Seeded synthetic MoE-layer workloads.

This module only draws inputs. It holds none of the layer's arithmetic (no
scoring, selection, permutation, expert MLP or combine), so both the CPU oracle
and the CUDA path can consume the same bytes from it.

Every tensor has its own seed, derived from the workload's base seed and a
fixed tensor id. Drawing one tensor therefore never shifts another, and a test
can draw only the logits of a large workload. Values come from torch's seeded
generator on the requested device. A tensor drawn on the GPU is copied to the
host whenever the oracle needs it, so both sides always see identical bytes.

Recipe (one line per tensor; std means standard deviation):
  logits    fp32 [T,E]   N(0,1), plus the per-expert skew bias where the
                          workload has one, or quantised to multiples of 0.5
  x         bf16 [T,H]   N(0,1), rounded to bf16 (round to nearest even)
  w_gate_up bf16 [E,H,2I] N(0, std 1/sqrt(H)); columns [0,I) gate, [I,2I) up
  w_down    bf16 [E,I,H] N(0, std 1/sqrt(I))
  shared_*  the same recipe for the one shared expert (E=1)
  dout      bf16 [T,H]   N(0,1), upstream gradient of the layer output
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1

# tensor ids: part of each tensor's seed
_TID = {"logits": 1, "x": 2, "w_gate_up": 3, "w_down": 4, "shared_gate_up": 5,
        "shared_down": 6, "dout": 7, "skew_rank": 8}


@dataclasses.dataclass(frozen=True)
class MoEWorkload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    score: int = SCORE_SOFTMAX
    renormalize: bool = True
    shared_expert: bool = False
    backward: bool = False
    skew: bool = False          # per-expert bias 3*ln(1/rank) and 16 dead experts
    dead_experts: int = 0
    tie_quantum: float = 0.0    # > 0: logits rounded to multiples of this
    seed: int = 1234

    @property
    def A(self) -> int:
        """Routed rows: every token is sent to exactly k experts (dropless)."""
        return self.T * self.k

    def fwd_flops(self) -> float:
        """Algorithmic expert-MLP FLOPs of one forward: 2*A*H*2I + 2*A*I*H."""
        f = 6.0 * self.A * self.H * self.I
        if self.shared_expert:
            f += 6.0 * self.T * self.H * self.I
        return f

    def bwd_flops(self) -> float:
        """Backward of the grouped MLP: dgrad and wgrad of both GEMMs."""
        return 12.0 * self.A * self.H * self.I

    def scaled(self, **kw) -> "MoEWorkload":
        return dataclasses.replace(self, **kw)


# The workloads, by model family. Shapes and distributions as stated in the
# recipe above.
WORKLOADS = {
    "tiny": MoEWorkload("tiny", T=64, H=128, I=256, E=8, k=2, seed=1234),
    "mixtral_8x7b": MoEWorkload("mixtral_8x7b", T=4096, H=4096, I=14336, E=8, k=2,
                                seed=1235),
    "qwen3_30b_a3b": MoEWorkload("qwen3_30b_a3b", T=4096, H=2048, I=768, E=128, k=8,
                                 backward=True, seed=1236),
    "llama4_17bx16e": MoEWorkload("llama4_17bx16e", T=8192, H=5120, I=8192, E=16, k=1,
                                  score=SCORE_SIGMOID, renormalize=False,
                                  shared_expert=True, seed=1237),
}
for _t in (1, 8, 64, 16384):
    WORKLOADS[f"skew_t{_t}"] = MoEWorkload(f"skew_t{_t}", T=_t, H=2048, I=768, E=128, k=8,
                                          skew=True, dead_experts=16, seed=1238 + _t)
WORKLOADS["tie_t64"] = MoEWorkload("tie_t64", T=64, H=2048, I=768, E=128, k=8,
                                   tie_quantum=0.5, seed=1300)


def _gen(w: MoEWorkload, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 64 + _TID[name])
    return g


def _normal(w, name, shape, device, std=1.0, dtype=torch.float32):
    g = _gen(w, name, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def skew_bias(w: MoEWorkload, device="cpu") -> torch.Tensor:
    """Per-expert logit bias of the skewed workloads: 3*ln(1/rank_e) over a
    seeded random ranking (rank 1..E), and -1e4 on the `dead_experts` experts
    with the largest rank, so that those receive no token."""
    g = _gen(w, "skew_rank", "cpu")
    perm = torch.randperm(w.E, generator=g)              # perm[e] + 1 = rank of e
    rank = (perm + 1).to(torch.float64)
    bias = 3.0 * torch.log(1.0 / rank)
    if w.dead_experts:
        bias[perm >= w.E - w.dead_experts] -= 1e4
    return bias.to(torch.float32).to(device)


def make_logits(w: MoEWorkload, device="cpu") -> torch.Tensor:
    l = _normal(w, "logits", (w.T, w.E), device)
    if w.skew:
        l = l + skew_bias(w, device)[None, :]
    if w.tie_quantum > 0:
        l = torch.round(l / w.tie_quantum) * w.tie_quantum   # round half to even
    return l.contiguous()


def make_x(w: MoEWorkload, device="cpu") -> torch.Tensor:
    return _normal(w, "x", (w.T, w.H), device, dtype=torch.bfloat16)


def make_w_gate_up(w: MoEWorkload, device="cpu") -> torch.Tensor:
    out = torch.empty((w.E, w.H, 2 * w.I), dtype=torch.bfloat16, device=device)
    g = _gen(w, "w_gate_up", device)
    std = 1.0 / math.sqrt(w.H)
    for e in range(w.E):          # per expert: bounded fp32 temporary
        out[e] = (torch.randn((w.H, 2 * w.I), generator=g, device=device) * std).to(torch.bfloat16)
    return out


def make_w_down(w: MoEWorkload, device="cpu") -> torch.Tensor:
    out = torch.empty((w.E, w.I, w.H), dtype=torch.bfloat16, device=device)
    g = _gen(w, "w_down", device)
    std = 1.0 / math.sqrt(w.I)
    for e in range(w.E):
        out[e] = (torch.randn((w.I, w.H), generator=g, device=device) * std).to(torch.bfloat16)
    return out


def make_shared(w: MoEWorkload, device="cpu"):
    if not w.shared_expert:
        return None, None
    gu = (_normal(w, "shared_gate_up", (1, w.H, 2 * w.I), device) / math.sqrt(w.H)).to(torch.bfloat16)
    d = (_normal(w, "shared_down", (1, w.I, w.H), device) / math.sqrt(w.I)).to(torch.bfloat16)
    return gu, d


def make_dout(w: MoEWorkload, device="cpu") -> torch.Tensor:
    return _normal(w, "dout", (w.T, w.H), device, dtype=torch.bfloat16)


def make_inputs(w: MoEWorkload, device="cpu", with_dout: Optional[bool] = None) -> dict:
    """All inputs of one workload on `device`."""
    d = {
        "logits": make_logits(w, device),
        "x": make_x(w, device),
        "w_gate_up": make_w_gate_up(w, device),
        "w_down": make_w_down(w, device),
    }
    d["shared_gate_up"], d["shared_down"] = make_shared(w, device)
    if with_dout is None:
        with_dout = w.backward
    if with_dout:
        d["dout"] = make_dout(w, device)
    return d
