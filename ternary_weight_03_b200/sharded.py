"""A ternary linear layer sharded over the output rows N, one GPU per rank.

The layer's rows are independent -- y[m, n] depends on row n of T only -- so
G ranks split N into contiguous slices: rank r keeps rows [b_r, e_r) of the
packed matrix (a packed row slice is the packing of the row slice, nothing
is repacked), X is replicated, each rank computes its columns Y[:, b_r:e_r]
with the library's kernels (tl_gemv / tl_gemm), and one all-gather assembles
Y on every rank.  This is the split that lets a model too large for one GPU's
memory run on several ("Pith review of Spectra 1.1", Figure 3, GPUs versus
relative speed-up, and the extension's 70B-on-one-GPU comparison).

The all-gather is torch.distributed's (NCCL over NVLink between GPUs; gloo on
CPU for the tests).  Every rank takes the same collective steps in the same
order; slices are padded to one common width so the gather moves equal
blocks, and each rank's block lands at its own column offset.
"""
from __future__ import annotations

import torch

import ternary_weight_03_b200 as tl


def slice_width(N: int, world: int, align: int = 8) -> int:
    """Common slice width: ceil(N / world) rounded up to a multiple of `align`
    (fp16 output rows then start on 16-byte boundaries)."""
    if N < 1 or world < 1 or align < 1:
        raise ValueError("N, world and align must be positive")
    per = -(-N // world)
    return -(-per // align) * align


def row_range(N: int, world: int, rank: int, align: int = 8) -> tuple[int, int]:
    """Rows [b, e) of rank `rank`: contiguous, in rank order, covering [0, N)
    exactly once; trailing ranks may get an empty slice when N is small."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    w = slice_width(N, world, align)
    b = min(N, rank * w)
    return b, min(N, b + w)


def gather_columns(y_local: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """All-gather the ranks' column slices [M, e_r - b_r] into Y [M, N], the
    same on every rank (rank r's block at columns [b_r, e_r))."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    M = y_local.shape[0]
    w = slice_width(N, world)
    b, e = row_range(N, world, rank)
    if y_local.shape[1] != e - b:
        raise ValueError(f"rank {rank}: local slice has {y_local.shape[1]} columns, expected {e - b}")
    block = torch.zeros((M, w), dtype=y_local.dtype, device=y_local.device)
    block[:, :e - b] = y_local
    blocks = [torch.empty_like(block) for _ in range(world)]
    dist.all_gather(blocks, block.contiguous(), group=group)
    out = torch.empty((M, N), dtype=y_local.dtype, device=y_local.device)
    for r in range(world):
        rb, re = row_range(N, world, r)
        out[:, rb:re] = blocks[r][:, :re - rb]
    return out


class ShardedLinear:
    """Rank-local part of an N-sharded layer: the packed rows of this rank
    live on its GPU; forward(X) returns the full Y [M, N] on every rank."""

    def __init__(self, fmt: int, packed_rows: torch.Tensor, alpha: float, N: int, K: int,
                 group=None):
        import torch.distributed as dist
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        self.b, self.e = row_range(N, world, rank)
        if packed_rows.shape[0] != self.e - self.b:
            raise ValueError(f"rank {rank} holds {packed_rows.shape[0]} rows, expected "
                             f"{self.e - self.b} (rows [{self.b}, {self.e}))")
        if packed_rows.shape[0] and not packed_rows.is_cuda:
            raise ValueError("packed rows must be on this rank's GPU")
        self.fmt, self.P, self.alpha, self.N, self.K, self.group = fmt, packed_rows, alpha, N, K, group

    def forward(self, X: torch.Tensor) -> torch.Tensor:
        M = X.shape[0]
        if self.e > self.b:
            y = tl.linear(self.fmt, self.P, self.alpha, X, self.K)
        else:
            y = torch.empty((M, 0), dtype=torch.float16, device=X.device)
        return gather_columns(y, self.N, self.group)
