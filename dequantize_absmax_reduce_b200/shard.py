"""Data-parallel sharding of the quantize path (one process per GPU).

Every group of every granularity except per-tensor lies inside one row of
the tensors these ops see, so row shards run with no exchange at all. Scales
that cover the whole tensor (per-tensor scaling, the NVFP4 per-tensor scale)
need the range of every shard: each rank writes its range record with
bq_group_range, the records are combined with one all-reduce MAX over int64
(the records hold IEEE bits of non-negative values, which order like
integers), and each rank quantizes its rows FROM_RANGE. Over NCCL that is a
16-byte all-reduce per tensor.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def row_range(n_rows: int, world: int, rank: int):
    """Contiguous, balanced row shard [start, stop) of rank `rank`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world / rank")
    base, extra = divmod(n_rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_ranges_(ranges: torch.Tensor, group=None) -> torch.Tensor:
    """In-place element-wise MAX of int64 range records across ranks."""
    if ranges.dtype != torch.int64:
        raise TypeError("range records are int64")
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(ranges, op=dist.ReduceOp.MAX, group=group)
    return ranges


def quantize_per_tensor_sharded(x_local: torch.Tensor, qdtype=torch.int8, symmetric=True,
                                group=None, **kw):
    """Per-tensor quantize of a row-sharded tensor: local range, one
    all-reduce MAX of the 16-byte record, local codes with the global scale."""
    from . import api
    r = api.group_range(x_local, "tensor")
    allreduce_ranges_(r, group)
    return api.quantize(x_local, "tensor", qdtype=qdtype, symmetric=symmetric, ranges=r, **kw)


def nvfp4_quantize_sharded(x_local: torch.Tensor, group=None):
    """NVFP4 of a row-sharded weight with the per-tensor scale of the whole tensor."""
    from . import _bq as B
    from . import api
    r = api.group_range(x_local, "tensor")
    allreduce_ranges_(r, group)
    n, k = x_local.shape
    packed = torch.empty((n, k // 2), dtype=torch.uint8, device=x_local.device)
    sc = torch.empty((n, k // 16), dtype=torch.uint8, device=x_local.device)
    s2 = torch.empty(1, dtype=torch.float32, device=x_local.device)
    B.bq_nvfp4_quantize(x_local, packed, sc, s2, 2, r)
    return packed, sc, s2
