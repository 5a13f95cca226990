"""Seeded synthetic workloads for the dMoE layer.

This module holds only the shapes and the seeded random inputs; it contains none of the
layer's arithmetic, so both the CUDA path and the CPU oracle can take their inputs from it.

Recipe: workload seed s = 1000 + workload number; every tensor has its own torch CPU
generator seeded with 100*s + i (i = 0 x, 1 W1, 2 W3, 3 W2, 4 logits, 5 dy, 6 W_r), so any
tensor can be regenerated alone; each is drawn in fp32 and rounded to bf16
(round-to-nearest-even):
  x ~ N(0, 1)                         [T, hidden]
  W1, W3 ~ 0.02 * N(0, 1)             [E, ffn, hidden]   (out, in) layout; W1 = gate
  W2 ~ 0.02 * N(0, 1)                 [E, hidden, ffn]
  logits ~ N(0, 1) (+ bias_e)         [T, E]
  dy ~ N(0, 1)                        [T, hidden]        (backward workloads only)
  W_r ~ N(0, 1) / sqrt(hidden)        [E, hidden]        (router weight, router runs only:
                                                          x W_r^T then has N(0, 1) logits)
The skewed workload adds bias_e = -1.5 * ln(e + 1) (Zipf-like skew toward low expert ids) to
the logits in fp32 before the bf16 rounding.  Std 0.02 matches the issue's
``init_method_std: 0.02``.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    number: int
    name: str
    T: int
    hidden: int
    ffn: int
    E: int
    top_k: int
    backward: bool = False
    zipf_bias: bool = False

    @property
    def seed(self) -> int:
        return 1000 + self.number

    @property
    def entries(self) -> int:
        return self.T * self.top_k

    def useful_flops(self, backward: bool | None = None) -> int:
        """Useful (unpadded) GEMM FLOPs: 6*N*h*f forward, +12*N*h*f backward."""
        b = self.backward if backward is None else backward
        f = 6 * self.entries * self.hidden * self.ffn
        return f + (12 * self.entries * self.hidden * self.ffn if b else 0)

    def describe(self) -> str:
        return (f"T={self.T} hidden={self.hidden} ffn={self.ffn} E={self.E} top_k={self.top_k}"
                f"{' zipf' if self.zipf_bias else ''}{' fwd+bwd' if self.backward else ' fwd'}")


WORKLOADS = {
    1: Workload(1, "tiny", 256, 128, 128, 8, 2),
    2: Workload(2, "mixtral_shaped", 4096, 4096, 14336, 8, 2),
    3: Workload(3, "fine_grained", 4096, 2048, 1024, 64, 8),
    4: Workload(4, "high_granularity", 16384, 1536, 256, 128, 8),
    5: Workload(5, "skewed_fwd_bwd", 32768, 2048, 512, 256, 8, backward=True, zipf_bias=True),
}


def custom(T, hidden, ffn, E, top_k, number=0, backward=False, zipf_bias=False, name="custom"):
    return Workload(number, name, T, hidden, ffn, E, top_k, backward, zipf_bias)


def zipf_bias(E: int) -> torch.Tensor:
    return torch.tensor([-1.5 * math.log(e + 1) for e in range(E)], dtype=torch.float32)


TENSORS = ("x", "w1", "w3", "w2", "logits", "dy", "w_router")


def make_tensor(w: Workload, name: str, seed: int | None = None) -> torch.Tensor:
    """One CPU bf16 input tensor of workload ``w`` (see the module recipe)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(100 * (w.seed if seed is None else seed) + TENSORS.index(name))
    shape, scale = {
        "x": ((w.T, w.hidden), 1.0),
        "w1": ((w.E, w.ffn, w.hidden), 0.02),
        "w3": ((w.E, w.ffn, w.hidden), 0.02),
        "w2": ((w.E, w.hidden, w.ffn), 0.02),
        "logits": ((w.T, w.E), 1.0),
        "dy": ((w.T, w.hidden), 1.0),
        "w_router": ((w.E, w.hidden), 1.0 / math.sqrt(w.hidden)),
    }[name]
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    if name == "logits" and w.zipf_bias:
        t += zipf_bias(w.E)[None, :]
    return t.to(torch.bfloat16)


def make_inputs(w: Workload, seed: int | None = None, with_dy: bool | None = None,
                with_router: bool = False) -> dict:
    """CPU bf16 tensors x, w1, w3, w2, logits (and dy, and the router weight w_router) for
    workload ``w``."""
    names = list(TENSORS[:5])
    if w.backward if with_dy is None else with_dy:
        names.append("dy")
    if with_router:
        names.append("w_router")
    return {n: make_tensor(w, n, seed) for n in names}
