"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds NO quantization or matmul arithmetic: it only draws random
bf16 tensors with the shapes and value structure of the workloads, on the CPU,
from seeded ``torch.Generator`` streams, so that the oracle and the CUDA path
see identical bytes.

Value structure (the pages' own workloads are Llama-2-7B/70B-shaped linear
layers; no model weights or datasets are used, these draws stand in for them):
  * weights  W[N, K] ~ N(0, sigma), optionally with a fraction of input channels
    (columns of W) multiplied by a factor (weight outliers);
  * activations X[M, K] ~ N(0, 1), optionally with a fraction of channels either
    multiplied by a factor or set to sign(x)·value (activation outliers of
    magnitude ≈100, the "|x|≈1 vs |x|≈100" example of "大模型推理中 Weight-only、
    W8A8 和 FP8 量化有什么区别？如何选型？", §三).
Outlier channel sets are ``randperm(K)[:round(frac·K)]`` from the same stream.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def make_weight(N: int, K: int, sigma: float, seed: int, outlier_frac: float = 0.0,
                outlier_scale: float = 1.0) -> torch.Tensor:
    """W[N, K] bf16 on the CPU: N(0, sigma) with optional scaled input channels."""
    g = _gen(seed)
    W = torch.randn(N, K, generator=g, dtype=torch.float32)
    W.mul_(sigma)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        ch = torch.randperm(K, generator=g)[:n_out]
        W[:, ch] *= outlier_scale
    return W.to(torch.bfloat16)


def make_activation(M: int, K: int, seed: int, outlier_frac: float = 0.0,
                    outlier_mode: str | None = None, outlier_value: float = 100.0) -> torch.Tensor:
    """X[M, K] bf16 on the CPU: N(0, 1) with optional outlier channels.

    outlier_mode "scale": chosen channels are multiplied by ``outlier_value``;
    outlier_mode "set":   chosen channels are set to sign(x)·``outlier_value``.
    """
    g = _gen(seed)
    X = torch.randn(M, K, generator=g, dtype=torch.float32)
    n_out = int(round(outlier_frac * K))
    if n_out > 0 and outlier_mode is not None:
        ch = torch.randperm(K, generator=g)[:n_out]
        if outlier_mode == "scale":
            X[:, ch] *= outlier_value
        elif outlier_mode == "set":
            sgn = torch.where(X[:, ch] >= 0, 1.0, -1.0)
            X[:, ch] = sgn * outlier_value
        else:
            raise ValueError(outlier_mode)
    return X.to(torch.bfloat16)


def make_act_scale(K: int, seed: int, lo: float = -1.5, hi: float = 1.5) -> torch.Tensor:
    """Per-input-channel activation scale a[K] (bf16), 2^u with u ~ U(lo, hi):
    positive factors of the size activation-aware scaling uses, with arbitrary
    bf16 mantissas (so x·a rounds).  Drawn on the CPU from its own seed."""
    g = _gen(seed)
    u = torch.rand(K, generator=g, dtype=torch.float32) * (hi - lo) + lo
    return torch.exp2(u).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(
        torch.bfloat16)


@dataclass(frozen=True)
class Layer:
    """One linear layer of a workload: Y[M, N] = X[M, K] · W[N, K]^T."""
    name: str
    K: int
    N: int
    sigma: float
    w_seed: int
    x_seed: int
    w_outlier_frac: float = 0.0
    w_outlier_scale: float = 1.0
    x_outlier_frac: float = 0.0
    x_outlier_mode: str | None = None
    x_outlier_value: float = 100.0

    def weight(self) -> torch.Tensor:
        return make_weight(self.N, self.K, self.sigma, self.w_seed, self.w_outlier_frac,
                           self.w_outlier_scale)

    def activation(self, M: int, seed_offset: int = 0) -> torch.Tensor:
        return make_activation(M, self.K, self.x_seed + seed_offset, self.x_outlier_frac,
                               self.x_outlier_mode, self.x_outlier_value)


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple
    Ms: tuple
    groups: tuple
    modes: tuple          # subset of ("asym", "sym")
    description: str = field(default="")


TINY = Workload(
    "tiny_w4a16_1x256x256",
    (Layer("tiny", K=256, N=256, sigma=0.02, w_seed=0, x_seed=1),),
    Ms=(1,), groups=(128,), modes=("asym",),
    description="M=1, K=256, N=256, g=128, asymmetric; W~N(0,0.02), X~N(0,1), seed 0")

DECODE_7B = Workload(
    "llama7b_shaped_decode",
    (Layer("up_4096x11008", K=4096, N=11008, sigma=0.02, w_seed=11, x_seed=12,
           w_outlier_frac=0.01, w_outlier_scale=20.0),
     Layer("down_11008x4096", K=11008, N=4096, sigma=0.02, w_seed=13, x_seed=14,
           w_outlier_frac=0.01, w_outlier_scale=20.0)),
    Ms=(1, 4, 16), groups=(128,), modes=("asym",),
    description="K=4096,N=11008 and K=11008,N=4096; M in {1,4,16}; g=128 asym; "
                "W~N(0,0.02) with 1% of input channels x20; X~N(0,1)")

DECODE_70B = Workload(
    "llama70b_shaped_decode",
    (Layer("up_8192x28672", K=8192, N=28672, sigma=0.015, w_seed=21, x_seed=22,
           x_outlier_frac=0.01, x_outlier_mode="set", x_outlier_value=100.0),
     Layer("down_28672x8192", K=28672, N=8192, sigma=0.015, w_seed=23, x_seed=24,
           x_outlier_frac=0.01, x_outlier_mode="set", x_outlier_value=100.0)),
    Ms=(1, 2, 8), groups=(128,), modes=("sym", "asym"),
    description="K=8192,N=28672 and K=28672,N=8192; M in {1,2,8}; g=128 sym and asym; "
                "W~N(0,0.015); X~N(0,1) with 1% of channels at sign(x)*100")

PREFILL = Workload(
    "prefill_2048x8192x8192",
    (Layer("prefill_8192x8192", K=8192, N=8192, sigma=0.02, w_seed=31, x_seed=32),),
    Ms=(2048,), groups=(128,), modes=("asym",),
    description="M=2048, K=N=8192, g=128 asym; W~N(0,0.02), X~N(0,1)")

CROSSOVER = Workload(
    "crossover_8192x8192",
    (Layer("cross_8192x8192", K=8192, N=8192, sigma=0.02, w_seed=41, x_seed=42,
           x_outlier_frac=0.01, x_outlier_mode="scale", x_outlier_value=100.0),),
    Ms=(1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 4096), groups=(32, 64, 128),
    modes=("sym", "asym"),
    description="K=N=8192; M in {1,...,4096}; g in {32,64,128}; sym and asym; "
                "W~N(0,0.02); X~N(0,1) with 1% of channels x100")

WORKLOADS = {w.name: w for w in (TINY, DECODE_7B, DECODE_70B, PREFILL, CROSSOVER)}
