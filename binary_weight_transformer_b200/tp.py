"""Tensor-parallel BitLinear layers over torch.distributed.

"M8.8 - Native Binary and Ternary Transformers" 0x08A-0x08C: when W is
sharded over ranks, global statistics (the per-tensor weight scale, the
per-token activation absmax, a norm's sum of squares) need a collective, and
row- and column-parallel layers own different scales.  The contract built
here is the global one: every rank's result equals the unsplit layer.

* Column-parallel (rank r owns output rows [n0, n1) of W): every rank takes
  the whole token rows x and computes its own output columns; the linear
  needs no collective.  The packed artifact is quantised once over the whole
  tensor (the ternary scale is per tensor, 0x05A) and sliced by rows, so the
  per-row scales (binary, 4-bit, OneBit's output vector h) are naturally
  local and the input-side vectors (the gain, OneBit's g) are replicated.
* Row-parallel (rank r owns input features [k0, k1)): the token statistics
  span the whole row, so each rank computes those of its slice, the maxima
  and the sums of squares are all-reduced, every slice takes its codes with
  the whole row's maximum, the int32 partial accumulators are all-reduced
  (integer addition is exact) and one epilogue rescales the sum.  The
  activation-side vectors are sliced with the features.

The page's own trace (0x08C) shows the other contract, group-local
quantisation with a float all-reduce of rescaled partial outputs; that is a
different method with its own checkpoint topology and is not what these
functions compute.

Every kernel is this library's (through the binding); the collectives are
torch.distributed's (NCCL between GPUs).  ``ops`` lets a test substitute the
per-rank compute (for example with the oracle on CPU ranks) to check the
partitioning and the order of the collectives.
"""
from __future__ import annotations

from types import SimpleNamespace

# Features per row-parallel slice are multiples of this, so that every
# slice of a packed row starts on a 16-byte boundary for all three formats
# (128 codes = 32, 16 and 64 bytes).
FEATURE_GRANULE = 128


def split(total: int, world: int, rank: int, granule: int = 1):
    """[start, stop) of rank `rank` when `total` items are split over `world`
    ranks in units of `granule` items, as evenly as possible."""
    if total % granule:
        raise ValueError(f"{total} is not a multiple of {granule}")
    units = total // granule
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start * granule, stop * granule


def feature_granule(hadamard: int = 0) -> int:
    return max(FEATURE_GRANULE, hadamard)


def packed_feature_slice(packed, fmt: int, k0: int, k1: int):
    """Columns of a packed artifact holding codes [k0, k1) of every row (a view
    with the same row stride); k0 and k1 multiples of FEATURE_GRANULE."""
    from . import BINARY1, INT4, TERNARY2
    if k0 % FEATURE_GRANULE or k1 % FEATURE_GRANULE:
        raise ValueError("slice bounds must be multiples of FEATURE_GRANULE")
    bits = {TERNARY2: 2, BINARY1: 1, INT4: 4}[fmt]
    return packed[:, k0 * bits // 8:k1 * bits // 8]


def row_scales_slice(s_w, fmt: int, n0: int, n1: int):
    """Weight scales of output rows [n0, n1): the per-tensor ternary scale
    as is, per-row scales sliced."""
    from . import TERNARY2
    return s_w if fmt == TERNARY2 else s_w[n0:n1]


def cuda_ops():
    """The per-rank compute of these layers: this library's kernels."""
    from . import (I32, lowbit_act_quant_given_max, lowbit_act_row_stats, lowbit_act_scales, lowbit_bitlinear,
                   lowbit_linear, lowbit_rescale)

    def linear_i32(q, s_x, packed, s_w, fmt, N, K):
        return lowbit_linear(q, s_x, packed, s_w, fmt, N, I32, K=K)

    return SimpleNamespace(row_stats=lowbit_act_row_stats, codes_given_max=lowbit_act_quant_given_max,
                           scales=lowbit_act_scales, linear_i32=linear_i32, rescale=lowbit_rescale,
                           bitlinear=lowbit_bitlinear)


def column_parallel_bitlinear(x, packed_rows, s_w_rows, fmt: int, n_local: int, out_dtype: int, g=None,
                              norm: int = 0, eps_norm: float = 1e-5, hadamard: int = 0, ops=None):
    """This rank's output columns y[:, n0:n1] from the whole token rows x and
    the packed rows [n0, n1) (no collective)."""
    ops = ops or cuda_ops()
    return ops.bitlinear(x, packed_rows, s_w_rows, fmt, n_local, out_dtype, g, norm, eps_norm, hadamard)


def gather_columns(y_local, group=None):
    """The full output from every rank's columns (all-gather, rank order)."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(y_local) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, y_local.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def row_parallel_bitlinear(x_local, packed_cols, s_w, fmt: int, N: int, K_total: int, out_dtype: int,
                           g_local=None, norm: int = 0, eps_norm: float = 1e-5, hadamard: int = 0, group=None,
                           ops=None):
    """The whole layer's output y [M, N] on every rank, from this rank's
    feature slice x_local [M, k1 - k0] and the packed columns of the same
    slice; equal to the unsplit layer (see the module doc)."""
    import torch.distributed as dist
    ops = ops or cuda_ops()
    K_local = x_local.shape[1]
    row_max, row_ss = ops.row_stats(x_local, g_local, hadamard, with_ss=bool(norm))
    dist.all_reduce(row_max, op=dist.ReduceOp.MAX, group=group)
    if norm:
        dist.all_reduce(row_ss, op=dist.ReduceOp.SUM, group=group)
    s_x = ops.scales(row_max, row_ss, K_total, norm, eps_norm, hadamard)
    q = ops.codes_given_max(x_local, row_max, g_local, hadamard)
    acc = ops.linear_i32(q, s_x, packed_cols, s_w, fmt, N, K_local)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return ops.rescale(acc, s_x, s_w, fmt, out_dtype)
