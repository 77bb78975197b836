"""Seeded synthetic workloads for the expert-choice MoE feed-forward layer.

This module only draws random numbers and shapes them. It holds none of the
layer's arithmetic, so both the CUDA path and the CPU oracle can consume its
output without sharing any computation.

The workloads follow NucleusMoE-Image's MoE FFN over patch tokens (NucleusMoE-Image
pipeline walkthrough, trdm.cn, section 1 "model positioning": a 1024 px image gives a
64x64 grid of patch tokens; section 4.3: classifier-free guidance runs a conditional
and an unconditional pass, so a CFG pair doubles the token count).

Recipe (fixed, so that every caller gets the same bytes):
  * one ``torch.Generator('cpu')`` per tensor, seeded ``seed + k`` with k fixed per
    tensor: x=0, W_r=1, W1=2, W3=3, W2=4, token scale=5, skew pieces=6..9;
  * x ~ N(0, 1); every weight ~ N(0, std = 1/sqrt(fan_in)) with fan_in = d for
    W_r, W1, W3 and F for W2 (LeCun-normal reading of "N(0, 1/sqrt(fan_in))");
  * the 1024 px workload multiplies each token row by s_t = exp(0.5 * n_t),
    n_t ~ N(0, 1) (LogNormal(0, 0.5));
  * the skewed workload builds W_r = U V^T / sqrt(4 d) + 0.1 G / sqrt(d) (rank 4 plus
    noise, so many experts prefer the same tokens) and gives 5% of the tokens
    (seeded choice) a row drawn from a pool of 32 integer-valued rows with entries
    in {-2..2}; tokens that share a pool row have bit-identical router logits and
    therefore exactly tied scores, which the layer breaks by lower token index;
  * everything is rounded once to the workload dtype (bf16 round-to-nearest-even,
    or kept fp32 for the fp32 workload).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    F: int
    capacity_factor: float
    dtype: str  # "bf16" or "f32"
    lognormal_scale: bool = False
    skewed: bool = False
    segments: int = 1  # selection runs per segment of T / segments tokens (per image)

    @property
    def C(self) -> int:
        # capacity per segment = ceil(capacity_factor * tokens / experts) (walkthrough
        # section 6.2, where a segment is one sample)
        return capacity(self.T // self.segments, self.capacity_factor, self.E)

    @property
    def Ce(self) -> int:
        """Entries per expert: C per segment."""
        return self.segments * self.C

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def expert_flops(self) -> float:
        # GEMM1 (gate + up) 4*E*C*d*F, GEMM2 2*E*C*F*d
        return 6.0 * self.E * self.Ce * self.d * self.F

    def router_flops(self) -> float:
        return 2.0 * self.T * self.d * self.E


def capacity(T: int, capacity_factor: float, E: int) -> int:
    return int(math.ceil(capacity_factor * T / E))


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny_fp32", T=256, d=256, E=8, F=512, capacity_factor=1, dtype="f32"),
        Workload("512px_cfg", T=2048, d=1024, E=16, F=2048, capacity_factor=2, dtype="bf16"),
        Workload("1024px_cfg", T=8192, d=2048, E=64, F=1024, capacity_factor=1, dtype="bf16",
                 lognormal_scale=True),
        Workload("batch4_1024px_cfg", T=32768, d=3072, E=64, F=1536, capacity_factor=4,
                 dtype="bf16"),
        Workload("skewed_2048px", T=16384, d=2048, E=128, F=768, capacity_factor=1,
                 dtype="bf16", skewed=True),
        # the model's own layer shape (walkthrough section 6 defaults: 128 experts of
        # width 1344, capacity factor 8) on a 1024 px CFG pair, selection per image
        Workload("model_default_1024px_cfg", T=8192, d=2048, E=128, F=1344,
                 capacity_factor=8, dtype="bf16", segments=2),
        # the batch-4 layer's expert GEMM shapes (2048 rows per expert, d = 3072, F = 1536)
        # with 16 experts instead of 64: the same kernels in ~1 GB of device memory, the
        # size for a full ncu capture of the tensor-bound GEMMs
        Workload("batch4_16experts", T=8192, d=3072, E=16, F=1536, capacity_factor=4,
                 dtype="bf16"),
    )
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal(shape, std: float, seed: int) -> torch.Tensor:
    return torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * std


def make_inputs(w: Workload, seed: int = 0, parts=("x", "W_r", "W1", "W3", "W2")) -> dict:
    """Return CPU tensors x [T,d], W_r [d,E], W1 [E,d,F], W3 [E,d,F], W2 [E,F,d].

    All tensors are contiguous, row-major and already rounded to ``w.torch_dtype``.
    ``parts`` limits which tensors are drawn (each has its own seed, so a subset has
    the same bytes as in the full set).
    """
    T, d, E, F = w.T, w.d, w.E, w.F
    x = _normal((T, d), 1.0, seed + 0)
    if w.lognormal_scale:
        s = torch.exp(0.5 * torch.randn(T, 1, generator=_gen(seed + 5), dtype=torch.float32))
        x = x * s
    if w.skewed:
        U = torch.randn(d, 4, generator=_gen(seed + 6), dtype=torch.float32)
        V = torch.randn(E, 4, generator=_gen(seed + 7), dtype=torch.float32)
        G = torch.randn(d, E, generator=_gen(seed + 8), dtype=torch.float32)
        W_r = U @ V.T / math.sqrt(4.0 * d) + 0.1 * G / math.sqrt(d)
        g9 = _gen(seed + 9)
        pool = torch.randint(-2, 3, (32, d), generator=g9).to(torch.float32)
        n_tied = max(1, int(round(0.05 * T)))
        who = torch.randperm(T, generator=g9)[:n_tied]
        which = torch.randint(0, 32, (n_tied,), generator=g9)
        x[who] = pool[which]
    else:
        W_r = _normal((d, E), 1.0 / math.sqrt(d), seed + 1)
    out = dict(x=x, W_r=W_r)
    if "W1" in parts:
        out["W1"] = _normal((E, d, F), 1.0 / math.sqrt(d), seed + 2)
    if "W3" in parts:
        out["W3"] = _normal((E, d, F), 1.0 / math.sqrt(d), seed + 3)
    if "W2" in parts:
        out["W2"] = _normal((E, F, d), 1.0 / math.sqrt(F), seed + 4)
    dt = w.torch_dtype
    return {k: v.to(dt).contiguous() for k, v in out.items() if k in parts}


def make_small(T: int, d: int, E: int, F: int, dtype: str = "f32", seed: int = 0,
               x_std: float = 1.0) -> dict:
    """Same recipe as :func:`make_inputs` for an arbitrary small shape (tests)."""
    w = Workload("custom", T=T, d=d, E=E, F=F, capacity_factor=1, dtype=dtype)
    out = make_inputs(w, seed)
    if x_std != 1.0:
        out["x"] = (out["x"].float() * x_std).to(w.torch_dtype)
    return out


def to_numpy_f64(t: torch.Tensor):
    """Exact widening of a bf16/fp32 CPU tensor to a float64 numpy array."""
    return t.detach().to(torch.float64).cpu().numpy()
