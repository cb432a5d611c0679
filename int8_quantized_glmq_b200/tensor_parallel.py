"""Tensor-parallel sharding of the quantized GLM-130B linear layers.

GLM-130B paper card (wikillm.com), "Paper vs code": the INT4 model runs 4-way
model-parallel (configs/model_glm_130b_int4.sh); the paper trains with 4-way tensor
parallelism. The usual split for a transformer layer:

  * column-parallel (QKV, FFN-up): rank r owns output rows [r N/T, (r+1) N/T) of the
    packed weight and its scales; Y is computed locally, [M, N/T] per rank, and may
    be all-gathered into [M, N];
  * row-parallel (attention output, FFN-down): rank r owns input columns
    [r K/T, (r+1) K/T) and the matching slice of X; each rank's output is a partial
    sum over its K range, and the ranks all-reduce it.

Quantize first, shard second: a layer is quantized once, whole, so every shard holds
exactly the codes and the per-row scales of the unsharded layer (a row-parallel
shard keeps the full row's scale). Column-parallel results are therefore identical
to the unsharded layer; row-parallel results differ only by the rounding of each
rank's fp16 partial output and of the fp16 sums of the all-reduce.

Biases (paper card, "Paper vs code": biases stay FP16) are fused into the local GEMM's
epilogue: a column-parallel shard takes the bias entries of its own rows (for a
GeGLU-packed FFN-up weight, the matching entries of both branches); a row-parallel
layer adds the bias on rank 0 only, so the reduced sum carries it once. A contiguous
shard of a GeGLU-packed weight (16-row groups) holds output columns
[rank F/T, (rank+1) F/T) of the GeGLU result, so its local output is again contiguous.

The collectives are torch.distributed ones on the tensors' device (NCCL between
GPUs). The local GEMM is the library's glmq_gemm_fused (through the binding) unless a
caller passes another function with the signature
``local(X, packed, scale, bits, bias, epilogue) -> Y``.
"""
from __future__ import annotations

from typing import Callable, Optional


def _dist():
    import torch.distributed as dist  # noqa: WPS433 (plumbing only)
    return dist


def _default_local():
    from ._binding import gemm, gemm_fused

    def local(X, packed, scale, bits, bias=None, epilogue="none"):
        if bias is None and epilogue == "none":
            return gemm(X, packed, scale, bits)
        return gemm_fused(X, packed, scale, bits, bias=bias, epilogue=epilogue)
    return local


def column_shard(packed, scale, rank: int, world: int):
    """(packed rows, scales) owned by ``rank`` in a column-parallel split (N % world == 0)."""
    N = packed.shape[0]
    if N % world != 0:
        raise ValueError(f"N={N} is not divisible by {world} ranks")
    n = N // world
    return packed[rank * n:(rank + 1) * n].contiguous(), scale[rank * n:(rank + 1) * n].contiguous()


def column_bias_shard(bias, rank: int, world: int, geglu: bool = False):
    """Bias entries (natural row order) of a column-parallel shard.

    For a GeGLU weight of 2F natural rows the shard's rows are F/T rows of the GELU
    branch followed by the same F/T rows of the gate branch."""
    N = bias.shape[0]
    if not geglu:
        n = N // world
        return bias[rank * n:(rank + 1) * n].contiguous()
    F = N // 2
    f = F // world
    import torch
    return torch.cat([bias[rank * f:(rank + 1) * f], bias[F + rank * f:F + (rank + 1) * f]]).contiguous()


def row_shard(packed, scale, bits: int, rank: int, world: int):
    """(packed columns, full scales) owned by ``rank`` in a row-parallel split.

    Each rank's K range must be a multiple of 64 values (the library's K rule)."""
    K = packed.shape[1] * 8 // bits
    if K % (64 * world) != 0:
        raise ValueError(f"K={K} cannot be split into {world} parts of a multiple of 64")
    kb = K // world * bits // 8                   # packed bytes per rank and row
    return packed[:, rank * kb:(rank + 1) * kb].contiguous(), scale


class ColumnParallelLinear:
    """Output rows [rank N/T, (rank+1) N/T) of a quantized linear layer.

    epilogue="geglu" takes a weight packed for the GeGLU epilogue (quantize with
    geglu=True); N/T must then be a multiple of 16."""

    def __init__(self, packed, scale, bits: int, rank: int, world: int, group=None,
                 bias=None, epilogue: str = "none", local: Optional[Callable] = None):
        if epilogue not in ("none", "geglu"):
            raise ValueError(f"unknown epilogue {epilogue!r}")
        if epilogue == "geglu" and (packed.shape[0] // world) % 16 != 0:
            raise ValueError("a GeGLU shard needs a multiple of 16 rows")
        self.packed, self.scale = column_shard(packed, scale, rank, world)
        self.bias = None if bias is None else column_bias_shard(bias, rank, world, epilogue == "geglu")
        self.bits, self.rank, self.world, self.group, self.epilogue = bits, rank, world, group, epilogue
        self.local = local or _default_local()

    def forward(self, X, gather: bool = False):
        """Y_local [M, N/T] (N/(2T) with GeGLU); with gather=True the full Y on every rank."""
        Y = self.local(X, self.packed, self.scale, self.bits, self.bias, self.epilogue)
        if not gather or self.world == 1:
            return Y
        import torch
        parts = [torch.empty_like(Y) for _ in range(self.world)]
        _dist().all_gather(parts, Y.contiguous(), group=self.group)
        return torch.cat(parts, dim=1)


def chunk_rows(N: int, chunks: int, align: int = 256):
    """Row ranges [(n0, n1), ...] splitting N output rows into about `chunks` pieces whose
    boundaries fall on multiples of `align` rows (the decode kernel's tile height)."""
    if N <= 0:
        return []
    per = -(-N // max(1, chunks))
    per = -(-per // align) * align
    return [(n0, min(N, n0 + per)) for n0 in range(0, N, per)]


class RowParallelLinear:
    """Input columns [rank K/T, (rank+1) K/T) of a quantized linear layer.

    forward() overlaps the reduction with the GEMM: the local GEMM runs in `chunks`
    pieces of output rows, and each piece's all-reduce is issued (asynchronously) as
    soon as its GEMM is enqueued, so the reduction of piece i runs while piece i+1 is
    computed (with NCCL the collective waits only for the work already on the stream).
    The pieces are reduced in fp16, the dtype the library writes: T - 1 fp16 roundings
    of the partial sums, within the accuracy bar of the layer. By default decode-sized
    inputs (M <= 16, where each piece would pay the GEMM's fixed cost) use one piece
    and larger M four."""

    def __init__(self, packed, scale, bits: int, rank: int, world: int, group=None,
                 bias=None, local: Optional[Callable] = None, chunks: Optional[int] = None):
        self.packed, self.scale = row_shard(packed, scale, bits, rank, world)
        self.K_local = self.packed.shape[1] * 8 // bits
        self.bias = bias if rank == 0 else None       # added once, by rank 0's epilogue
        self.bits, self.rank, self.world, self.group = bits, rank, world, group
        self.local = local or _default_local()
        self.chunks = chunks

    def local_input(self, X):
        """This rank's slice of a full activation X [M, K]."""
        return X[:, self.rank * self.K_local:(self.rank + 1) * self.K_local].contiguous()

    def partial(self, X_local, n0: int = 0, n1: Optional[int] = None):
        """This rank's fp16 partial output [M, n1 - n0] over its K range for output rows
        [n0, n1) (all rows by default); rank 0 adds the bias."""
        n1 = self.packed.shape[0] if n1 is None else n1
        bias = None if self.bias is None else self.bias[n0:n1]
        return self.local(X_local, self.packed[n0:n1], self.scale[n0:n1], self.bits, bias, "none")

    def forward(self, X_local, chunks: Optional[int] = None):
        """Y [M, N] on every rank: the fp16 partial outputs summed by the all-reduce."""
        if self.world == 1:
            return self.partial(X_local)
        M = X_local.shape[0]
        n = chunks or self.chunks or (1 if M <= 16 else 4)
        pieces, works = [], []
        for n0, n1 in chunk_rows(self.packed.shape[0], n):
            Y = self.partial(X_local, n0, n1)
            works.append(_dist().all_reduce(Y, group=self.group, async_op=True))
            pieces.append(Y)
        for w in works:
            w.wait()
        if len(pieces) == 1:
            return pieces[0]
        import torch
        return torch.cat(pieces, dim=1)
