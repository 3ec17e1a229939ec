"""Output-feature (N) sharded W4A16 linear layer across the ranks of a process group.

Weights too large for one GPU — the 70B-class layers whose FP16 weights take
140 GB against 35 GB in INT4 ("推理优化中“用精度换性能“的核心技术：量化", §1) —
are split by output feature: rank r holds rows [n0_r, n1_r) of W[N, K], quantizes
them (groups run along K inside a row, so a row's codes, scale and zero point do
not depend on the split) and multiplies them against the full X; one all-gather
of the per-rank Y slices over NCCL (NVLink/NVSwitch) assembles Y[M, N].  There
is no other exchange: the split is column-parallel in the GEMM's output.

Every rank computes the same number of rows (ceil(N / world)); the last rank's
slice is padded with nothing — it computes only the rows that exist and zero-
fills the rest of its gather buffer — so the collective moves equal-size
chunks, and the padding is dropped after the gather.

The local GEMM is the library's fused kernel (``w4a16.gemm``); it can be
replaced (``local_gemm=``) by any function with the same signature, which is
how the sharding and gather logic is exercised without GPUs.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def shard_rows(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [n0, n1) of an N-row weight owned by `rank` of `world`: contiguous
    slices of ceil(N / world) rows, the last ones shorter or empty."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    per = -(-N // world)
    n0 = min(rank * per, N)
    return n0, min(n0 + per, N)


def gather_columns(Y_local: torch.Tensor, N: int, world: int, group=None) -> torch.Tensor:
    """All-gather the per-rank Y slices [M, ceil(N/world)] (rows past N zero) and
    return Y[M, N] with rank r's slice in columns [r·per, (r+1)·per)."""
    import torch.distributed as dist
    M, per = Y_local.shape
    if world == 1:
        return Y_local[:, :N]
    # The collective concatenates along dim 0: gather [per, M] slices of Yᵀ so
    # that the result, transposed back, is Y with the slices side by side.
    send = Y_local.t().contiguous()
    recv = torch.empty((world * per, M), dtype=Y_local.dtype, device=Y_local.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    return recv[:N].t().contiguous()


class ShardedW4A16Linear:
    """This rank's slice of a W4A16 linear layer Y = X·Ŵᵀ, N sharded over `group`.

    Build with ``from_weight`` (quantizes this rank's rows of the full W) or
    with already quantized slice tensors.  ``forward(X)`` runs the local fused
    GEMM on the rank's rows and all-gathers Y[M, N] on every rank."""

    def __init__(self, N: int, K: int, g: int, sym: bool, packed, scales, zeros,
                 world: int = 1, rank: int = 0, group=None,
                 local_gemm: Optional[Callable] = None):
        self.N, self.K, self.g, self.sym = N, K, g, sym
        self.world, self.rank, self.group = world, rank, group
        self.n0, self.n1 = shard_rows(N, world, rank)
        self.per = -(-N // world)
        if packed.shape[0] != self.n1 - self.n0:
            raise ValueError(f"rank {rank} holds {packed.shape[0]} rows, expected {self.n1 - self.n0}")
        self.packed, self.scales, self.zeros = packed, scales, zeros
        if local_gemm is None:
            from . import gemm as local_gemm
        self.local_gemm = local_gemm

    @classmethod
    def from_weight(cls, W: torch.Tensor, g: int = 128, sym: bool = False, world: int = 1,
                    rank: int = 0, group=None, quantize: Optional[Callable] = None,
                    local_gemm: Optional[Callable] = None) -> "ShardedW4A16Linear":
        """Quantize rows [n0, n1) of the full W[N, K] (bf16) for this rank."""
        N, K = W.shape
        n0, n1 = shard_rows(N, world, rank)
        if quantize is None:
            from . import quantize
        P, S, Z = quantize(W[n0:n1].contiguous(), g, sym)
        return cls(N, K, g, sym, P, S, Z, world, rank, group, local_gemm)

    def forward(self, X: torch.Tensor) -> torch.Tensor:
        M = X.shape[0]
        rows = self.n1 - self.n0
        Y_local = torch.zeros((M, self.per), dtype=torch.bfloat16, device=X.device)
        if rows > 0:
            Y_local[:, :rows] = self.local_gemm(X, self.packed, self.scales, self.zeros, self.g,
                                                self.sym)
        return gather_columns(Y_local, self.N, self.world, self.group)

    __call__ = forward
