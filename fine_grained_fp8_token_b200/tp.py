"""Tensor-parallel column split of the W8A8 linear layer over P GPUs.

The pages run the layer on one GPU; this is the multi-GPU extension of it.
One process per GPU, torch.distributed (NCCL) for the plumbing.  The split
is along the weight's output channels:

  * rank r owns output channels [r * n, (r + 1) * n), n = N / P, in whole
    128-row blocks, so each 128x128 block keeps its scale: the rank's Wq / Ws
    are row slices of the full layer's (quantizing the rank's slice of W
    gives exactly those bytes);
  * activations are replicated: every rank quantizes the whole X (1x128
    groups along K do not depend on N) and runs fgfp8_linear on its slice,
    giving its part Y_r [M, n];
  * a plain all-gather brings the P parts into this GPU's memory as
    [P, M, n], and fgfp8_gather_cols writes them as Y [M, N].

No kernel is given another GPU's memory: the all-gather copies remote parts
into local memory first, and the library uses no multicast of any kind.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import SCALE_F32, gather_cols, linear, quant_weight, scale_rows

BLOCK = 128


def shard_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Output channels [n0, n1) of `rank` in a column split of N over `world`
    ranks.  Every rank gets the same whole number of 128-row blocks (the
    all-gather needs equal parts), so N must be a multiple of 128 * world."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} is not in a world of {world}")
    if N % (BLOCK * world) != 0:
        raise ValueError(f"N = {N} is not a multiple of 128 x {world} ranks")
    n = N // world
    return rank * n, (rank + 1) * n


def shard_weight(Wq, Ws, world: int, rank: int):
    """The rank's rows of a quantized weight: Wq [N, K] codes and Ws
    [N/128, K/128] block scales of the full layer -> (Wq[n0:n1],
    Ws[n0/128:n1/128]), contiguous views."""
    n0, n1 = shard_range(Wq.shape[0], world, rank)
    return Wq[n0:n1], Ws[n0 // BLOCK:n1 // BLOCK]


def all_gather_parts(Y_local, group=None):
    """All ranks' parts Y_r [M, n] stacked as [P, M, n] in this rank's
    memory (every rank takes this collective step, in the same order)."""
    import torch
    import torch.distributed as dist
    P = dist.get_world_size(group)
    parts = torch.empty((P,) + tuple(Y_local.shape), dtype=Y_local.dtype, device=Y_local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(parts.view(P * Y_local.shape[0], *Y_local.shape[1:]), Y_local.contiguous(),
                                    group=group)
    else:
        dist.all_gather(list(parts.unbind(0)), Y_local.contiguous(), group=group)
    return parts


@dataclass
class ColumnParallelLinear:
    """This rank's share of a W8A8 linear layer split along N.

    Wq, Ws: the rank's rows of the quantized weight (see shard_weight, or
    from_weight to quantize the rank's slice of a bf16 W).  forward(X) runs
    the quantizer and GEMM on the rank's slice, all-gathers the parts and
    returns the full Y [M, N] (bf16) on every rank."""
    Wq: object
    Ws: object
    fmt: int
    N: int
    group: object = None

    @classmethod
    def from_weight(cls, W, fmt: int = SCALE_F32, group=None):
        """Quantize this rank's rows of W bf16 [N, K] (all ranks hold W, or
        at least their rows of it, in the same full-layer indexing)."""
        import torch.distributed as dist
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        n0, n1 = shard_range(W.shape[0], world, rank)
        Wq, Ws = quant_weight(W[n0:n1], fmt)
        return cls(Wq, Ws, fmt, W.shape[0], group)

    def forward(self, X, Xq=None, Xs=None):
        import torch
        M, K = X.shape
        if Xq is None:
            Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
        if Xs is None:
            Xs = torch.empty((K // BLOCK, scale_rows(M, self.fmt)),
                             dtype=torch.float32 if self.fmt == SCALE_F32 else torch.uint8, device=X.device)
        Y_local = linear(X, self.Wq, self.Ws, self.fmt, Xq=Xq, Xs=Xs)
        parts = all_gather_parts(Y_local, self.group)
        return gather_cols(parts)
