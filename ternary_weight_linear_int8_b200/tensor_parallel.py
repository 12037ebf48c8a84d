"""Tensor-parallel BitNet FFN block over a torch.distributed process group.

For models whose FFN does not fit one GPU (the pages discuss 100B-class
models on CPUs -- dashen-tech.com "BitNet.cpp 深度解析" -- and 70B-class
serving -- abeam.tech review, section "推論コストはどれだけ下がったのか"), the
block is split over G ranks, one process per GPU:

* gate and up by rows: rank r holds intermediate features [i0, i1), whole
  groups of 64;
* down by the same features (its input columns), norm2_w likewise;
* every rank holds the whole token and the whole-matrix gammas.

Per block: the gate/up step on every rank, an all-reduce (MAX) of the
per-token absmax of h' * n2 and one (SUM) of sum h'^2, the down step, an
exact int32 SUM all-reduce of the partial accumulators, and the finishing
dequantisation (include/bitnet.h, bitnet_ffn_tp_*).  The compute steps are
passed in as an ``ops`` object, so the same orchestration runs on the GPU
(``GpuFfnOps``, the library's kernels, NCCL) and in CPU tests.  Every rank
takes the same collectives in the same order.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

ALIGN = 64          # features per sharding unit (the kernels' K granularity)


def shard_bounds(I: int, world: int, rank: int, align: int = ALIGN):
    """Feature range [i0, i1) of ``rank``: whole groups of ``align``, split as
    evenly as the groups allow."""
    if I % align:
        raise ValueError(f"the intermediate width must be a multiple of {align}")
    groups = I // align
    if groups < world:
        raise ValueError("fewer feature groups than ranks")
    g0 = groups * rank // world
    g1 = groups * (rank + 1) // world
    return g0 * align, g1 * align


@dataclass
class FfnShard:
    """One rank's part of an FFN block (device tensors, packed I2_S codes)."""
    gate: torch.Tensor          # [i1 - i0, H/4]
    gamma_gate: torch.Tensor    # whole-matrix gamma
    up: torch.Tensor            # [i1 - i0, H/4]
    gamma_up: torch.Tensor
    down: torch.Tensor          # [H, (i1 - i0)/4]
    gamma_down: torch.Tensor
    norm1_w: torch.Tensor | None
    norm2_w: torch.Tensor | None   # [i1 - i0] or None
    I: int                      # whole intermediate width
    i0: int
    i1: int


def shard_packed_ffn(gate, gamma_gate, up, gamma_up, down, gamma_down, I, world, rank,
                     norm1_w=None, norm2_w=None) -> FfnShard:
    """Slice whole packed matrices (packed with their whole-matrix gammas)
    into this rank's shard."""
    i0, i1 = shard_bounds(I, world, rank)
    return FfnShard(
        gate=gate[i0:i1].contiguous(), gamma_gate=gamma_gate,
        up=up[i0:i1].contiguous(), gamma_up=gamma_up,
        down=down[:, i0 // 4:i1 // 4].contiguous(), gamma_down=gamma_down,
        norm1_w=norm1_w, norm2_w=None if norm2_w is None else norm2_w[i0:i1].contiguous(),
        I=I, i0=i0, i1=i1)


class GpuFfnOps:
    """The per-shard steps on the library's CUDA kernels (argument
    marshalling only)."""

    def __init__(self, bitnet_module):
        self.B = bitnet_module

    def gate_up(self, x, s: FfnShard):
        return self.B.bitnet_ffn_tp_gate_up(x, s.gate, s.gamma_gate, s.up, s.gamma_up,
                                            s.norm1_w, s.norm2_w)

    def down(self, h, s: FfnShard, amax2):
        return self.B.bitnet_ffn_tp_down(h, s.down, amax2, s.norm2_w)

    def finish(self, acc, s: FfnShard, amax2, sumsq_x, sumsq_h, eps):
        return self.B.bitnet_ffn_tp_finish(acc, s.I, s.gamma_down, amax2, sumsq_x, sumsq_h,
                                           eps=eps, want_f32=True)


def tp_ffn(x, shard: FfnShard, ops, group=None, eps: float = 1e-5):
    """The FFN block on this rank's shard; every rank returns the whole
    output (y bf16 [M,H], y_f32)."""
    h, amax2, sumsq_h, sumsq_x = ops.gate_up(x, shard)
    dist.all_reduce(amax2, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(sumsq_h, op=dist.ReduceOp.SUM, group=group)
    acc = ops.down(h, shard, amax2)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return ops.finish(acc, shard, amax2, sumsq_x, sumsq_h, eps)
