"""Context parallelism for route-set QSA across GPUs (one process per GPU).

The layout is the pages' context-parallel one: each rank attends with its
local slice of query rows against the gathered global K/V, and route IDs stay
in global key coordinates ("flex_qsa" page, module description: context
parallelism is local queries against gathered global K/V; "fa4_qsa" page,
``fa4_sparse_gqa_attention``: the key tensor may hold gathered global K/V while
the query is a local CP slice).  Each rank owns

* a contiguous range of query rows (chosen by ``balanced_query_ranges`` so that
  every rank gets about the same number of routed pairs, the unit of work), and
* a contiguous, equal slice of the K/V rows (the keys it stores and whose
  gradients it returns).

Forward: all-gather the K/V slices (BF16), then the route-set forward of the
local queries.  Backward: all-gather again, run the backward with FP32 dK/dV
(each rank's queries contribute to keys anywhere in the sequence), and
reduce-scatter those FP32 partials so that every rank receives the summed
gradients of its own K/V slice, rounded to BF16 once.  The collectives are
``torch.distributed`` (NCCL over NVLink on GPUs); the attention itself is the
library's CUDA path.  With NCCL the all-gathers run on a side stream and the
library calls get their completion as an event: the route preprocessing, which
reads no K/V, runs under the gather, and only the first kernel that reads K/V
waits (qsa_forward_kvwait / qsa_backward_kvwait).  The local compute is a
parameter only so that the collective plumbing can be exercised on CPU
processes.
"""

from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist


def balanced_query_ranges(row_counts, world: int) -> list:
    """Contiguous query ranges [start, end) per rank, balanced by routed pairs.

    Rank r ends at the first row whose prefix sum of ``row_counts`` reaches
    (r + 1) / world of the total; empty rows ride along with their neighbours.
    """
    c = np.asarray(row_counts, dtype=np.int64)
    T = c.size
    if world < 1:
        raise ValueError("world must be >= 1")
    prefix = np.concatenate([[0], np.cumsum(c)])
    total = int(prefix[-1])
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        end = int(np.searchsorted(prefix, target, side="left"))
        bounds.append(min(max(end, bounds[-1]), T))
    bounds.append(T)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def kv_slice(T_kv: int, world: int, rank: int):
    """The contiguous K/V rows [start, end) that rank owns (equal slices)."""
    if T_kv % world != 0:
        raise ValueError("T_kv must be divisible by the number of ranks")
    n = T_kv // world
    return rank * n, (rank + 1) * n


def _all_gather_rows(x: torch.Tensor, group=None) -> torch.Tensor:
    world = dist.get_world_size(group)
    out = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    else:
        dist.all_gather(list(out.chunk(world)), x.contiguous(), group=group)
    return out


def _reduce_scatter_rows(x: torch.Tensor, group=None) -> torch.Tensor:
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n = x.shape[0] // world
    if dist.get_backend(group) == "nccl":
        out = torch.empty((n,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        dist.reduce_scatter_tensor(out, x.contiguous(), op=dist.ReduceOp.SUM, group=group)
        return out
    y = x.contiguous().clone()  # backends without reduce-scatter: all-reduce, keep the own slice
    dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y[rank * n:(rank + 1) * n].clone()


def _streamed(group, x: torch.Tensor) -> bool:
    """Whether the collectives run on CUDA streams (NCCL, device tensors)."""
    return x.is_cuda and dist.get_backend(group) == "nccl"


_SIDE_STREAMS = {}


def _side_stream(device):
    """One side stream per device for the all-gathers, created once: a fresh
    stream per call cost several ms per step over the first few dozen steps
    (one B200, world size 1: 15.4 ms against 7.9 ms once warm)."""
    key = torch.device(device).index
    if key not in _SIDE_STREAMS:
        _SIDE_STREAMS[key] = torch.cuda.Stream(device=device)
    return _SIDE_STREAMS[key]


def _gather_kv_async(k_local, v_local, group=None):
    """All-gathers K and V on a side stream; returns ``(k, v, ready)`` where the
    event ``ready`` fires once both are complete.  Nothing on the current
    stream waits for it: the caller hands it to the library call."""
    main = torch.cuda.current_stream(k_local.device)
    side = _side_stream(k_local.device)
    side.wait_stream(main)  # the local slices are written on the current stream
    with torch.cuda.stream(side):
        k = _all_gather_rows(k_local, group)
        v = _all_gather_rows(v_local, group)
        ready = torch.cuda.Event()
        ready.record(side)
    for t in (k, v):  # allocated on the side stream, read on the current one
        t.record_stream(main)
    for t in (k_local, v_local):
        t.record_stream(side)
    return k, v, ready


def cp_forward(q, k_local, v_local, routes, scale: float, group=None, local_forward=None, workspace=None):
    """Forward of this rank's query rows against the gathered global K/V.

    ``q`` [T_local, H, d] and ``routes`` [T_local, n_sel] (global key IDs) are the
    rank's query rows; ``k_local`` / ``v_local`` [T_kv / world, G, d] its K/V
    slice.  Returns ``(out, lse)`` of the local rows.  ``workspace`` (optional)
    is the library forward's workspace; passed on to ``cp_backward`` as
    ``saved_workspace`` it spares the backward the route sort.
    """
    if local_forward is None:
        from . import qsa
        if _streamed(group, k_local):
            k, v, ready = _gather_kv_async(k_local, v_local, group)
            return qsa.forward(q, k, v, routes, scale, kv_ready=ready, workspace=workspace)
        if workspace is not None:
            def local_forward(q_, k_, v_, r_, s_):
                return qsa.forward(q_, k_, v_, r_, s_, workspace=workspace)
        else:
            local_forward = qsa.forward
    k = _all_gather_rows(k_local, group)
    v = _all_gather_rows(v_local, group)
    return local_forward(q, k, v, routes, scale)


def cp_backward(grad_out, q, k_local, v_local, out, lse, routes, scale: float, group=None, local_backward=None,
                final_cast=None, saved_workspace=None):
    """Backward of this rank's query rows; returns ``(dq, dk_local, dv_local)``.

    dq covers the local query rows; dk_local / dv_local are the gradients of the
    rank's own K/V slice summed over every rank's queries (FP32 reduce-scatter,
    then one rounding to BF16 by the library's cast kernel).  ``local_backward``
    must return FP32 (or wider) dK/dV partials; ``final_cast(x)`` rounds the
    rank's summed slice (both are parameters only so that the collective
    plumbing can run on CPU processes).  ``saved_workspace``: the workspace
    given to ``cp_forward`` for the same rows (its route lists are reused).
    """
    if local_backward is None or final_cast is None:
        from . import qsa
    if final_cast is None:
        final_cast = qsa.cast_f32_to_bf16
    if local_backward is None and _streamed(group, k_local):
        k, v, ready = _gather_kv_async(k_local, v_local, group)
        dq, dk_part, dv_part = qsa.backward(grad_out, q, k, v, out, lse, routes, scale, kv_fp32=True,
                                            kv_ready=ready, saved_workspace=saved_workspace)
    else:
        if local_backward is None:
            def local_backward(go, q_, k_, v_, o_, l_, r_, s_):
                return qsa.backward(go, q_, k_, v_, o_, l_, r_, s_, kv_fp32=True, saved_workspace=saved_workspace)
        k = _all_gather_rows(k_local, group)
        v = _all_gather_rows(v_local, group)
        dq, dk_part, dv_part = local_backward(grad_out, q, k, v, out, lse, routes, scale)
    if dk_part.dtype not in (torch.float32, torch.float64) or dv_part.dtype != dk_part.dtype:
        raise TypeError("local_backward must return FP32 (or FP64) dK/dV partials")
    dk = final_cast(_reduce_scatter_rows(dk_part, group))
    dv = final_cast(_reduce_scatter_rows(dv_part, group))
    return dq, dk, dv
