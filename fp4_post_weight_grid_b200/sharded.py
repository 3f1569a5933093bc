"""Row-sharded quantization of one weight across the ranks of a process group.

Blocks never cross a row, so a weight split by rows quantizes independently on
each rank, with one exception: the NVFP4 global scale S = max|x| / (256*6)
(ScaleSweep summary, "Metodologia: ScaleSweep" sec. 2) is a property of the
whole weight.  The only exchange is therefore one all-reduce (MAX) of a single
float before the sweep; MXFP4 needs none.  Each rank's result equals the rows
it owns of the single-device quantization.

The exchange protocol (`row_shard_protocol`) is written against three
callables so that the host logic can be exercised without a GPU; the product
entry point (`nvfp4_quantize_row_shard`) binds them to the CUDA library and
`torch.distributed` (NCCL over NVLink on a GPU node).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch


def shard_rows(rows: int, world: int, rank: int) -> Tuple[int, int]:
    """[start, stop) of the rows owned by `rank` when `rows` rows are split as
    evenly as possible over `world` ranks (the first rows % world ranks get one
    more)."""
    if world < 1 or not 0 <= rank < world or rows < 0:
        raise ValueError(f"bad split: rows={rows} world={world} rank={rank}")
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def row_shard_protocol(local_absmax: Callable[[], torch.Tensor],
                       all_reduce_max: Callable[[torch.Tensor], None],
                       sweep: Callable[[torch.Tensor], object]):
    """The row-sharded NVFP4 exchange: the local max of |x| (a one-element
    float tensor), its all-reduce to the maximum over all ranks, then the sweep
    of the local rows with that global max.  Returns what `sweep` returns."""
    amax = local_absmax()
    all_reduce_max(amax)
    return sweep(amax)


def nvfp4_quantize_row_shard(w_shard: torch.Tensor, group=None, importance: Optional[torch.Tensor] = None,
                             with_deq: bool = True, with_loss: bool = True, stream=None):
    """NVFP4 ScaleSweep of this rank's rows of a weight split by rows across
    the ranks of `group` (every rank calls it, with its own rows; the row
    counts may differ, the column count may not).  Returns an NVFP4Result whose
    amax and global_scale are those of the whole weight."""
    import torch.distributed as dist

    from . import (NVFP4_BLOCK, NVFP4Result, _rc, fp4q_global_absmax, fp4q_nvfp4_sweepmse,
                   fp4q_nvfp4_sweepwmse)

    rows, cols = _rc(w_shard, NVFP4_BLOCK)
    dev = w_shard.device
    kw = dict(device=dev)
    S = torch.empty(1, dtype=torch.float32, **kw)
    status = torch.zeros(1, dtype=torch.int32, **kw)
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, **kw)
    scales = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.uint8, **kw)
    deq = torch.empty_like(w_shard) if with_deq else None
    loss = torch.empty((rows, cols // NVFP4_BLOCK), dtype=torch.float32, **kw) if with_loss else None

    def local_absmax():
        amax = torch.empty(1, dtype=torch.float32, **kw)
        fp4q_global_absmax(w_shard, amax, stream=stream)
        return amax

    def all_reduce_max(amax):
        if stream is not None:
            torch.cuda.current_stream(dev).wait_stream(stream)
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream(dev))

    def sweep(amax):
        if importance is None:
            fp4q_nvfp4_sweepmse(w_shard, amax, codes, scales, S, deq, loss, status, stream)
        else:
            fp4q_nvfp4_sweepwmse(w_shard, amax, importance, codes, scales, S, deq, loss, status, stream)
        return NVFP4Result(codes, scales, S, deq, loss, amax, status)

    return row_shard_protocol(local_absmax, all_reduce_max, sweep)
