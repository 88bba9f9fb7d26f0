"""Tensor-parallel TTQ projections: one layer split over the GPUs of a
process group (NCCL), one process per GPU.

The pages describe TTQ on one GPU (TTQ review, "Proposed method"); this
module splits one quantized projection the way a tensor-parallel linear
layer is split, and adds only the exchange that TTQ itself needs.

Column-parallel (the output rows of W are split). Every rank holds all of
X, so the statistics and scales of X are computed on every rank; the
deterministic kernels give every rank the same s. Each rank quantizes its
rows of W and projects; TTQ needs no collective. ``gather=True`` all-gathers
the output columns.

Row-parallel (the input channels are split, on group boundaries, so no
group straddles two ranks). Rank p holds channels [k0_p, k1_p) of X and W.
The statistics are local, but the shrinkage mean runs over all channels
(bullet 3, C_lambda): each rank forms its shard's channel total, one
all-reduce of one fp64 scalar adds them, and each rank takes its scales
with that mean. Each rank then quantizes its columns of W and projects in
fp32; an all-reduce adds the partial outputs, which are rounded to the
output type last.

``ops`` is the module whose calls run the steps: the CUDA binding
(test_weight_quantization_b200.ttq) by default. Tests of the host logic
pass a stand-in with the same calls.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ttq as _ttq


def shard_channels(K: int, world: int, group: int) -> list[tuple[int, int]]:
    """[k0, k1) input-channel ranges of a row-parallel split: near-equal,
    every boundary a multiple of lcm(group, 32) so that groups and 32-code
    blocks stay whole. Raises ValueError when K cannot be split so."""
    unit = group if group % 32 == 0 else 32
    if K % unit != 0:
        raise ValueError(f"K = {K} is not a multiple of {unit}")
    units = K // unit
    if units < world:
        raise ValueError(f"K = {K} has fewer than {world} units of {unit}")
    b = [unit * (units * i // world) for i in range(world + 1)]
    return [(b[i], b[i + 1]) for i in range(world)]


def shard_rows(N: int, world: int) -> list[tuple[int, int]]:
    """[n0, n1) output-row ranges of a column-parallel split (near-equal)."""
    if N < world:
        raise ValueError(f"N = {N} has fewer rows than {world} ranks")
    b = [N * i // world for i in range(world + 1)]
    return [(b[i], b[i + 1]) for i in range(world)]


class RowParallelTTQLinear:
    """The projection Y = X W^T with W's input channels split over the
    ranks of ``group`` (this rank holds ``W_shard`` = W[:, k0:k1] and is
    called with X[:, k0:k1])."""

    def __init__(self, W_shard: torch.Tensor, K_total: int,
                 params: "_ttq.TTQParams", group=None, ops=None):
        self.ops = ops or _ttq
        self.W = W_shard
        self.K_total = int(K_total)
        self.params = params
        self.group = group
        K = W_shard.shape[1]
        if K % params.group != 0 or K % 32 != 0:
            raise ValueError("a shard must hold whole groups and 32-code "
                             "blocks")

    def __call__(self, X_shard: torch.Tensor,
                 out_dtype=torch.bfloat16) -> torch.Tensor:
        ops, prm = self.ops, self.params
        T = X_shard.shape[0]
        sums = ops.act_stats(X_shard, prm.p)
        total = ops.channel_moment_total(sums, T)
        dist.all_reduce(total, op=dist.ReduceOp.SUM, group=self.group)
        s, inv = ops.awq_scales_sharded(sums, T, self.K_total, total,
                                        prm.alpha, prm.lam, prm.p)
        c, d, z = ops.quantize_rtn_grouped(self.W, s, prm.bits, prm.group)
        Y = ops.w_lowbit_gemm(X_shard, inv, c, d, z, self.W.shape[0],
                              prm.bits, prm.group, out_dtype=torch.float32)
        dist.all_reduce(Y, op=dist.ReduceOp.SUM, group=self.group)
        return Y if out_dtype == torch.float32 else Y.to(out_dtype)


class ColumnParallelTTQLinear:
    """The projection Y = X W^T with W's output rows split over the ranks
    of ``group`` (this rank holds ``W_shard`` = W[n0:n1, :] and is called
    with all of X)."""

    def __init__(self, W_shard: torch.Tensor, params: "_ttq.TTQParams",
                 group=None, ops=None):
        self.ops = ops or _ttq
        self.W = W_shard
        self.params = params
        self.group = group

    def __call__(self, X: torch.Tensor, gather: bool = False,
                 out_dtype=torch.bfloat16) -> torch.Tensor:
        ops, prm = self.ops, self.params
        T = X.shape[0]
        sums = ops.act_stats(X, prm.p)
        s, inv = ops.awq_scales(sums, T, prm.alpha, prm.lam, prm.p)
        c, d, z = ops.quantize_rtn_grouped(self.W, s, prm.bits, prm.group)
        Y = ops.w_lowbit_gemm(X, inv, c, d, z, self.W.shape[0], prm.bits,
                              prm.group, out_dtype=out_dtype)
        if not gather:
            return Y
        world = dist.get_world_size(self.group)
        sizes = [torch.zeros(1, dtype=torch.int64, device=Y.device)
                 for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([Y.shape[1]], dtype=torch.int64,
                                            device=Y.device),
                        group=self.group)
        parts = [torch.empty((T, int(n.item())), dtype=Y.dtype,
                             device=Y.device) for n in sizes]
        dist.all_gather(parts, Y.contiguous(), group=self.group)
        return torch.cat(parts, dim=1)
