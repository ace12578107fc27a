"""Tensor-parallel quantized linear layers over torch.distributed.

[wiki] "ZSE - open-source движок для запуска LLM локально на GPU - 2026",
section "Тензорный параллелизм": the weights are sharded across processes (one
per GPU), column-parallel for the QKV / Gate / Up projections and row-parallel
for O / Down, and the processes exchange results through NCCL collectives.

* Column-parallel: shard r keeps output rows [n_r, n_{r+1}) of W -- a row range
  of the packed codes, scales and zeros, taken without a copy -- and computes
  its M x N_r slice of y with zq_linear.  No exchange is needed when the next
  layer is row-parallel (it consumes exactly that slice).
* Row-parallel: shard r keeps the columns of whole groups [g_r, g_{r+1}) of 128
  (copied once into their own N x K_r tensors) and receives the matching
  columns of x; zq_linear_partial gives its fp32 partial sums of the full
  M x N output.  The shards' partial sums are added and rounded once to fp16
  by zq_reduce_partials, either in rank order after an all-gather ("ordered":
  the same bits on every rank, whatever P) or after NCCL's all-reduce
  ("all_reduce": NCCL's own order).

The shard planner and the exchanges are host logic (plain torch.distributed
calls on whatever tensors they are given); every step of the arithmetic runs
in the library's kernels.
"""
import torch

from . import (GROUP, ZQ_ERR_INVALID_ARG, ZQError, linear, linear_partial, zq_reduce_partials)

ROW_ALIGN = 64  # rows per shard boundary: keeps every shard's row blocks whole and its pointers aligned


def row_shard(N, P, r, align=ROW_ALIGN):
    """Output rows [n0, n1) of column-parallel shard r of P: whole blocks of
    `align` rows, as even as possible (the last block may be short)."""
    if not (0 <= r < P) or N <= 0:
        raise ZQError(ZQ_ERR_INVALID_ARG, f"row_shard: N={N}, P={P}, r={r}")
    units = -(-N // align)
    u0, u1 = r * units // P, (r + 1) * units // P
    return min(u0 * align, N), min(u1 * align, N)


def group_shard(K, P, r, group=GROUP):
    """Input columns [k0, k1) of row-parallel shard r of P: whole groups, as
    even as possible."""
    if K % group != 0 or not (0 <= r < P):
        raise ZQError(ZQ_ERR_INVALID_ARG, f"group_shard: K={K} (a multiple of {group}), P={P}, r={r}")
    G = K // group
    return (r * G // P) * group, ((r + 1) * G // P) * group


def column_shard(packed, scales, zeros, N, K, bits, P, r):
    """Views of the packed codes, scales and zeros of shard r's rows (no copy);
    returns ((packed, scales, zeros), (n0, n1))."""
    n0, n1 = row_shard(N, P, r)
    words = K * bits // 32
    p = packed.reshape(N, words)[n0:n1]
    s = scales.reshape(N, K // GROUP)[n0:n1]
    z = zeros.reshape(N, K // GROUP)[n0:n1]
    return (p, s, z), (n0, n1)


def k_shard(packed, scales, zeros, N, K, bits, P, r):
    """Shard r's groups as their own contiguous tensors (a group of 128 codes
    is exactly 4*bits words of its row, so the slice is whole words); returns
    ((packed N x K_r*bits/32, scales N x G_r, zeros N x G_r), (k0, k1))."""
    k0, k1 = group_shard(K, P, r)
    words = K * bits // 32
    w0, w1 = k0 * bits // 32, k1 * bits // 32
    g0, g1 = k0 // GROUP, k1 // GROUP
    p = packed.reshape(N, words)[:, w0:w1].contiguous()
    s = scales.reshape(N, K // GROUP)[:, g0:g1].contiguous()
    z = zeros.reshape(N, K // GROUP)[:, g0:g1].contiguous()
    return (p, s, z), (k0, k1)


def _world(group):
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def gather_partials(part, group=None):
    """Every rank's fp32 partial sums, in rank order (all-gather)."""
    import torch.distributed as dist
    world, _ = _world(group)
    if world == 1:
        return [part]
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part.contiguous(), group=group)
    return parts


def all_reduce_partials(part, group=None):
    """The sum of every rank's fp32 partial sums, in place (NCCL's order)."""
    import torch.distributed as dist
    world, _ = _world(group)
    if world > 1:
        dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return part


class ColumnParallelLinear:
    """Shard r of a column-parallel quantized linear layer: output rows
    [n0, n1) of W."""

    def __init__(self, packed, scales, zeros, N, K, bits, rank, world):
        (self.packed, self.scales, self.zeros), (self.n0, self.n1) = column_shard(
            packed, scales, zeros, N, K, bits, world, rank)
        self.N, self.K, self.bits = self.n1 - self.n0, K, bits

    def forward(self, x, out=None, stream=None):
        """x: fp16 M x K (every rank the same) -> this rank's fp16 M x (n1 - n0) slice of y."""
        if self.N == 0:
            return torch.empty(x.shape[0], 0, dtype=torch.float16, device=x.device)
        return linear(x, self.packed, self.scales, self.zeros, self.bits, self.N, out=out, stream=stream)


class RowParallelLinear:
    """Shard r of a row-parallel quantized linear layer: input columns
    [k0, k1) (whole groups) of W."""

    def __init__(self, packed, scales, zeros, N, K, bits, rank, world):
        (self.packed, self.scales, self.zeros), (self.k0, self.k1) = k_shard(
            packed, scales, zeros, N, K, bits, world, rank)
        self.N, self.K, self.bits = N, self.k1 - self.k0, bits

    def partial(self, x_shard, stream=None):
        """fp32 partial sums (M x N) of this shard: x_shard is M x (k1 - k0)."""
        if self.K == 0:
            return torch.zeros(x_shard.shape[0], self.N, dtype=torch.float32, device=x_shard.device)
        return linear_partial(x_shard, self.packed, self.scales, self.zeros, self.bits, self.N, stream=stream)

    def forward(self, x_shard, group=None, mode="ordered", stream=None):
        """fp16 M x N output on every rank: this shard's partial sums, the
        exchange (`mode` "ordered" or "all_reduce"), then one fp16 rounding."""
        part = self.partial(x_shard, stream)
        if mode == "ordered":
            parts = gather_partials(part, group)
        elif mode == "all_reduce":
            parts = [all_reduce_partials(part, group)]
        else:
            raise ZQError(ZQ_ERR_INVALID_ARG, f"mode must be 'ordered' or 'all_reduce', got {mode!r}")
        y = torch.empty(part.shape, dtype=torch.float16, device=part.device)
        zq_reduce_partials(parts, part.numel(), y, stream)
        return y
