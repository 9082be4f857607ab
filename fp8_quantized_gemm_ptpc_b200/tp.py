"""Tensor-parallel PTPC-FP8 linear layers over ``torch.distributed``.

The PTPC page ("PTPC-FP8: boosting vLLM performance on AMD ROCm") evaluates
its models with tensor parallelism (TP = 2, benchmark section).  A linear
layer splits over ranks in two ways, and PTPC's scales behave differently in
each:

* Column-parallel (the output channels Co split): rank r holds the weight
  columns ``[o0, o1)`` with their per-channel scales, which depend only on
  those columns, and the whole activation.  Per-token quantisation reads the
  whole row, so every rank computes the same codes and scales, and its output
  columns are those of the unsplit layer.  No collective, unless the caller
  wants the full output gathered.

* Row-parallel (the input channels Ci split): rank r holds the slice
  ``X[:, k0:k1]`` and weight rows ``[k0, k1)``.  A token's scale comes from
  its whole row, so the ranks all-reduce their slice row maxima (MAX, T
  floats, exact in any order) and quantise their slice with the combined
  maxima; codes and scales equal the unsplit ones.  The weight codes are the
  unsplit per-output-channel codes (each column's scale is over all Ci),
  sliced along K.  Each rank computes the unscaled fp32 partial accumulator
  ``acc_r[t, o] = sum_{k in slice} dec(Xq) dec(Wq)``; the accumulators are
  all-reduced (SUM) and the rank-1 scale ``(acc * x_scale[t]) * w_scale[o]``
  and the bf16 rounding are applied once to the sum.  The result differs from
  the unsplit layer only in the fp32 summation order.

The arithmetic goes through an ``ops`` object: :class:`CudaOps` is the
library's sm_100a kernels (the product path); a test can pass another
implementation of the same seven methods to check the partitioning on CPU
ranks.  Collectives go through ``torch.distributed`` (NCCL between GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n: int, rank: int, world: int, align: int = 16):
    """[start, stop) of rank's share of n items, cut at multiples of `align`
    (the library's 16-element row rule; 128 for sub-byte weights).  Shares
    differ by at most `align` items; ranks past the end get empty shares."""
    if n % align != 0:
        raise ValueError(f"{n} is not a multiple of {align}")
    blocks = n // align
    per, extra = divmod(blocks, world)
    start = rank * per + min(rank, extra)
    stop = start + per + (1 if rank < extra else 0)
    return start * align, stop * align


class CudaOps:
    """The library's kernels, on CUDA tensors (the product path)."""

    def __init__(self, ptpc=None):
        if ptpc is None:
            import fp8_quantized_gemm_ptpc_b200 as ptpc
        self.p = ptpc

    def quantize_weights(self, W):
        return self.p.quantize_weights(W)

    def linear(self, X, Wq_t, w_scale):
        return self.p.linear(X, Wq_t, w_scale)

    def row_amax(self, X):
        return self.p.row_amax(X)

    def quantize_activations_amax(self, X, amax):
        return self.p.quantize_activations_amax(X, amax)

    def unscaled_mm(self, Xq, Wq_t):
        return self.p.unscaled_mm_f32(Xq, Wq_t)

    def apply_scales(self, acc, x_scale, w_scale):
        return self.p.apply_scales(acc, x_scale, w_scale)

    def slice_k(self, Wq_t, k0, k1):
        return Wq_t[:, k0:k1].contiguous()


class ColumnParallelLinear:
    """Output channels [o0, o1) of a PTPC-FP8 linear layer on this rank.

    ``W`` is the full bf16 weight [Ci, Co] (as a checkpoint loader has it);
    this rank quantises only its columns, whose scales depend on nothing
    else.  ``forward(X)`` takes the whole activation and returns this rank's
    output columns, or, with ``gather=True``, all of them (all-gather)."""

    def __init__(self, W: torch.Tensor, rank: int, world: int, ops=None, group=None):
        self.ops = ops or CudaOps()
        self.group = group
        self.world = world
        Ci, self.Co = W.shape
        self.o0, self.o1 = shard_range(self.Co, rank, world)
        if self.o1 == self.o0:
            raise ValueError(f"{self.Co} output channels do not give every one of {world} ranks a share")
        self.Wq_t, self.w_scale = self.ops.quantize_weights(W[:, self.o0:self.o1].contiguous())

    def forward(self, X: torch.Tensor, gather: bool = False) -> torch.Tensor:
        out = self.ops.linear(X, self.Wq_t, self.w_scale)
        if not gather or self.world == 1:
            return out
        # shares may differ by one 16-channel block: gather equal-width
        # (padded) pieces and trim each to its rank's share
        spans = [shard_range(self.Co, r, self.world) for r in range(self.world)]
        width = max(b - a for a, b in spans)
        mine = torch.zeros((X.shape[0], width), dtype=out.dtype, device=out.device)
        mine[:, :out.shape[1]] = out
        parts = [torch.empty_like(mine) for _ in spans]
        dist.all_gather(parts, mine, group=self.group)
        return torch.cat([p[:, :b - a] for p, (a, b) in zip(parts, spans)], dim=1)


class RowParallelLinear:
    """Input channels [k0, k1) of a PTPC-FP8 linear layer on this rank.

    ``W`` is the full bf16 weight [Ci, Co]: it is quantised per output
    channel over all Ci (the unsplit codes and scales) and this rank keeps
    the codes of its K slice.  ``forward(X_r)`` takes this rank's activation
    slice X[:, k0:k1] and returns the whole bf16 output [T, Co], identical on
    every rank (two all-reduces: the row maxima, then the accumulators)."""

    def __init__(self, W: torch.Tensor, rank: int, world: int, ops=None, group=None):
        self.ops = ops or CudaOps()
        self.group = group
        self.world = world
        Ci, Co = W.shape
        self.k0, self.k1 = shard_range(Ci, rank, world)
        if self.k1 == self.k0:
            raise ValueError(f"{Ci} input channels do not give every one of {world} ranks a share")
        Wq_t, self.w_scale = self.ops.quantize_weights(W)
        self.Wq_t = self.ops.slice_k(Wq_t, self.k0, self.k1)

    # The three phases of forward, between which the ranks exchange data.
    def slice_amax(self, X_r: torch.Tensor) -> torch.Tensor:
        """Row maxima of this rank's slice (to be combined with MAX)."""
        return self.ops.row_amax(X_r)

    def partial(self, X_r: torch.Tensor, amax: torch.Tensor):
        """Codes of the slice with the combined maxima, and the slice's
        unscaled partial accumulator (to be combined with SUM); also returns
        the token scales, which equal the unsplit ones."""
        Xq, x_scale = self.ops.quantize_activations_amax(X_r, amax)
        return self.ops.unscaled_mm(Xq, self.Wq_t), x_scale

    def finish(self, acc: torch.Tensor, x_scale: torch.Tensor) -> torch.Tensor:
        """The rank-1 scale and the bf16 rounding of the summed accumulator."""
        return self.ops.apply_scales(acc, x_scale, self.w_scale)

    def forward(self, X_r: torch.Tensor) -> torch.Tensor:
        amax = self.slice_amax(X_r)
        if self.world > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.group)
        acc, x_scale = self.partial(X_r, amax)
        if self.world > 1:
            dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
        return self.finish(acc, x_scale)
