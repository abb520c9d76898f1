"""Expert parallelism of the decode layer across GPUs, one process per GPU.

The routed experts are split into contiguous ranges, one per rank; rank 0 also
owns the shared expert.  Every rank routes every token (the router is
replicated, so the selection is the same bits everywhere), runs the FFN of the
union experts in its own range only -- its expert table may leave every other
entry NULL -- and produces a partial output

    out_r[t] = [rank 0: y_shared(t)] + sum over s with idx[t,s] in range_r of w[t,s] * y_s(t).

One exchange step, an all-reduce (sum) of out[T][H] over the group, gives the
layer's output on every rank.  This is the GPU form of the pages' cluster mode,
where the dense part stays on a coordinator and the routed FFNs run on workers
(colibri deep review page, its local-cluster section); here every rank holds
its share of the experts in HBM, which multiplies the expert capacity by the
number of GPUs.  The partial sums are added in another order than the
single-GPU combine, so the result agrees with it within the layer's float
tolerance, not bit for bit.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import MoeDims, _arg, _check, _ptr, _rows, _stream, lib


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """The routed experts [lo, hi) that `rank` of `world` owns: contiguous,
    disjoint, covering [0, E), sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world or E < 1:
        raise ValueError(f"bad partition: E={E}, world={world}, rank={rank}")
    return rank * E // world, (rank + 1) * E // world


def owns_shared(rank: int) -> bool:
    """The shared expert's FFN runs on rank 0 only (it is added once)."""
    return rank == 0


def partial_layer_forward(d: MoeDims, x, Wr, table, out, ws, expert_lo: int, expert_hi: int,
                          with_shared: bool, route_counts=None, stream=None) -> None:
    """One rank's share of the layer (moe_layer_forward_ep): routing of every
    token, the FFNs of the union experts in [expert_lo, expert_hi) and of the
    shared expert if with_shared, and their weighted sum into out [T][H].
    Table entries outside the range are never read."""
    T = _rows(x, "x", d.H)
    _arg(Wr, "Wr", torch.float32, d.E * d.H)
    _arg(table, "table", torch.int64, d.E + 1)
    _arg(out, "out", torch.float32, T * d.H)
    _arg(ws, "ws", torch.uint8)
    _arg(route_counts, "route_counts", torch.int32, d.E, optional=True)
    _check("moe_layer_forward_ep", lib().moe_layer_forward_ep(
        ctypes.byref(d), T, _ptr(x), _ptr(Wr), _ptr(table), _ptr(out), _ptr(ws), ws.numel(),
        _ptr(route_counts), int(expert_lo), int(expert_hi), 1 if with_shared else 0, _stream(stream)))


def reduce_partials(out: torch.Tensor, group=None) -> torch.Tensor:
    """The exchange step: out <- sum of every rank's partial output (in place)."""
    import torch.distributed as dist
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def layer_forward_ep(d: MoeDims, x, Wr, table, out, ws, group=None, route_counts=None, stream=None) -> None:
    """The whole layer on the ranks of `group` (default: the world): this
    rank's partial output, then the all-reduce; every rank ends with the
    layer's output in out."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    lo, hi = expert_range(d.E, world, rank)
    partial_layer_forward(d, x, Wr, table, out, ws, lo, hi, owns_shared(rank), route_counts, stream)
    reduce_partials(out, group)
