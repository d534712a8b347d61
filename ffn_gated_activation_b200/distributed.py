"""Multi-GPU plumbing for SiTU-GLU: one process per GPU over torch.distributed.

Rows are independent (each output row depends on its own gate_up row, weight
and grad_out row only), so:

* Data parallelism shards rows -- contiguous blocks, ``shard_range`` -- and
  needs no collective for row-aligned routing weights.
* A routing weight broadcast to every row has one gradient for all rows: its
  per-rank partials are summed across ranks (``allreduce_drw``).
* Tensor parallelism of FC1 (column-parallel: rank r holds gate columns
  [a_r, b_r) and the matching up columns, see ``tp_local_gate_up``) keeps the
  forward and dG/dU local; a row-aligned or broadcast routing-weight
  gradient, a sum over all I columns, needs the sum of the ranks' partial
  sums over their columns: an all-reduce of T values (``situ_glu_bwd_tp``).
  Per-column ([I]) and per-element ([..., I]) weights are sharded with their
  columns (``tp_local_columns``); their gradients stay local.
* Under data parallelism a per-column weight is shared by every row shard,
  so its [I] gradient is all-reduced like a broadcast weight's.
* An NVFP4 output has one per-tensor scale.  When a tensor is split over the
  ranks of a tensor-parallel group (column shards of Y or d_gate_up), every
  shard must be coded with the maximum of the whole tensor: each rank
  computes its shard's maximum, the maxima are all-reduced (MAX), and each
  rank codes its shard with the result (``situ_glu_fwd_nvfp4_tp``,
  ``situ_glu_bwd_nvfp4_tp``).  Column shards of a block-scaled tensor keep
  whole blocks (``align`` = 16 for NVFP4, 32 for MXFP8).  Row shards under
  data parallelism are separate tensors and keep their own scales.

Nothing here computes the method; the kernels run in libsitu_glu.so.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import functional


def shard_range(n: int, rank: int, world: int, align: int = 1) -> tuple[int, int]:
    """Contiguous [start, stop) of ``n`` items for ``rank`` of ``world``: sizes
    differ by at most ``align`` and every boundary is a multiple of ``align``
    (except ``n`` itself)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if align <= 0:
        raise ValueError("align must be positive")
    units = -(-n // align)
    base, extra = divmod(units, world)
    start_u = rank * base + min(rank, extra)
    stop_u = start_u + base + (1 if rank < extra else 0)
    return min(n, start_u * align), min(n, stop_u * align)


def vector_width(dtype: torch.dtype) -> int:
    """Elements per 16-byte vector: the granularity a column shard keeps."""
    return 16 // torch.empty((), dtype=dtype).element_size()


def tp_local_gate_up(gate_up: torch.Tensor, rank: int, world: int, align: int | None = None) -> torch.Tensor:
    """The [..., 2 * I_r] gate_up a column-parallel FC1 produces on ``rank``:
    gate columns [a, b) followed by the same up columns [I + a, I + b).
    Shard boundaries are multiples of ``align`` (default: one 16-byte vector)."""
    inter = gate_up.shape[-1] // 2
    a, b = shard_range(inter, rank, world, align or vector_width(gate_up.dtype))
    return torch.cat([gate_up[..., a:b], gate_up[..., inter + a:inter + b]], dim=-1).contiguous()


def tp_local_columns(x: torch.Tensor, rank: int, world: int, align: int | None = None) -> torch.Tensor:
    """Columns [a, b) of an [..., I] tensor (grad_out or Y) held by ``rank``."""
    a, b = shard_range(x.shape[-1], rank, world, align or vector_width(x.dtype))
    return x[..., a:b].contiguous()


def allreduce_drw(d_rw: torch.Tensor, group=None) -> torch.Tensor:
    """Sum routing-weight gradient partials over ``group`` in place (NCCL for
    CUDA tensors, gloo for CPU tensors)."""
    dist.all_reduce(d_rw, op=dist.ReduceOp.SUM, group=group)
    return d_rw


def situ_glu_bwd_tp(gate_up_local, routing_weights, grad_out_local, beta=functional.DEFAULT_BETA,
                    linear_beta=functional.DEFAULT_LINEAR_BETA, group=None, want_drw=True, **kw):
    """Backward of a column-parallel shard: local d_gate_up [..., 2 I_r] and the
    routing-weight gradient.  Row-aligned and broadcast weights span every
    column, so their partials are all-reduced over ``group``; per-column and
    per-element weights are passed as this rank's columns and their gradient
    is already complete."""
    lead = tuple(gate_up_local.shape[:-1])
    inter_local = gate_up_local.shape[-1] // 2
    with _on_stream(kw.pop("stream", None)):  # the kernel, then the all-reduce of its result, on one stream
        d_gate_up, d_rw = functional.situ_glu_bwd(gate_up_local, routing_weights, grad_out_local, beta,
                                                  linear_beta, want_drw=want_drw, **kw)
        if d_rw is not None and tp_drw_needs_allreduce(lead, inter_local, routing_weights):
            allreduce_drw(d_rw, group)
    return d_gate_up, d_rw


def _on_stream(stream):
    """Context that makes ``stream`` current (no-op for None)."""
    import contextlib
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def allreduce_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """Largest of the ranks' tensor maxima, in place (the per-tensor scale of a
    tensor whose shards live on the ranks of ``group``)."""
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def situ_glu_fwd_nvfp4_tp(gate_up_local, routing_weights, beta=functional.DEFAULT_BETA,
                          linear_beta=functional.DEFAULT_LINEAR_BETA, group=None, **kw):
    """NVFP4 forward of a column-parallel shard (gate_up_local from
    ``tp_local_gate_up(..., align=16)``): the shard's maximum, the group's
    maximum, then the shard's codes under the whole tensor's scale.  Returns
    (data, scale, amax) as situ_glu_fwd_nvfp4."""
    with _on_stream(kw.pop("stream", None)):  # the three steps in order on one stream
        _, _, amax = functional.situ_glu_fwd_nvfp4(gate_up_local, routing_weights, beta, linear_beta,
                                                   amax_only=True)
        allreduce_amax(amax, group)
        return functional.situ_glu_fwd_nvfp4(gate_up_local, routing_weights, beta, linear_beta, amax=amax, **kw)


def situ_glu_bwd_nvfp4_tp(gate_up_local, routing_weights, grad_out_local, beta=functional.DEFAULT_BETA,
                          linear_beta=functional.DEFAULT_LINEAR_BETA, group=None, want_drw=True, **kw):
    """NVFP4 backward of a column-parallel shard: d_gate_up's codes under the
    whole tensor's scale (the group's maximum of the shards' maxima), and the
    routing-weight gradient all-reduced as in ``situ_glu_bwd_tp``.  Returns
    (data, scale, amax, d_rw) as situ_glu_bwd_nvfp4."""
    with _on_stream(kw.pop("stream", None)):
        _, _, amax, _ = functional.situ_glu_bwd_nvfp4(gate_up_local, routing_weights, grad_out_local, beta,
                                                      linear_beta, amax_only=True)
        allreduce_amax(amax, group)
        data, scale, amax, d_rw = functional.situ_glu_bwd_nvfp4(gate_up_local, routing_weights, grad_out_local,
                                                                beta, linear_beta, want_drw=want_drw, amax=amax, **kw)
        lead = tuple(gate_up_local.shape[:-1])
        if d_rw is not None and tp_drw_needs_allreduce(lead, gate_up_local.shape[-1] // 2, routing_weights):
            allreduce_drw(d_rw, group)
    return data, scale, amax, d_rw


def tp_drw_needs_allreduce(lead: tuple, inter_local: int, routing_weights) -> bool:
    """Whether a column-parallel shard's routing-weight gradient is a partial
    sum (row-aligned or broadcast weights) rather than this rank's own slice
    (per-column or per-element weights)."""
    from . import abi
    mode = functional.routing_mode(lead, inter_local, routing_weights)[0]
    return mode in (abi.SITU_RW_ROW, abi.SITU_RW_SCALAR)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Largest ``value`` over the ranks (timing: a step lasts as long as its
    slowest rank).  Returns ``value`` when no process group is initialised."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
