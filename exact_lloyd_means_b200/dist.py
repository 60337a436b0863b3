"""Data-parallel Lloyd's k-means over several GPUs (one process per GPU).

The rows of X are split across the ranks of a torch.distributed process group and the
centroids are replicated.  Each iteration:

  1. every rank assigns its own rows (fk_assign),
  2. every rank reduces its rows to per-cluster fp64 sums, counts and its share of the
     objective (fk_update_partial),
  3. the ranks exchange those with one all_gather per tensor (NCCL over NVLink on GPUs;
     any backend works),
  4. every rank combines the gathered shards in rank order (fk_finalize_shards): the same
     bits on every rank, whatever the number of ranks' reduction order would otherwise be.

Only step 3 is communication; steps 1, 2 and 4 are the library's kernels.  The local
steps are passed in as a `LocalOps` object so the exchange logic can be exercised with any
backend, including gloo ranks on CPU with stand-in local steps.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist


@dataclass
class LocalOps:
    """The per-rank steps of a run.

    prepare(X)  (optional) once per run, before the first assignment
    assign(X, C) -> labels
    partial(X, labels, C) -> (sums [K, d] fp64, counts [K] int64, objective [1] fp64)
    finalize(sums_w [W, K, d], counts_w [W, K], objs_w [W], C_old) ->
        (C_new, counts [K] int64, objective [1] fp64)
    """
    assign: Callable
    partial: Callable
    finalize: Callable
    prepare: Optional[Callable] = None


def gpu_ops(N: int, d: int, K: int, dtype, device) -> LocalOps:
    """LocalOps backed by libfk on one GPU, for N local points of dimension d and K
    centroids (workspace and outputs allocated once).  For fp32 points, prepare() splits
    them into their bf16 hi/lo planes once per run (as fk_lloyd does once per call)
    instead of on every assignment; the points must not change during the run."""
    from . import fk
    ws = fk.workspace(N, d, K, dtype, "l2", device=device)
    planes = fk.split_points_buffer(N, d, device) if dtype == torch.float32 else None
    state = {"x": None, "split": None}
    labels = torch.empty(N, dtype=torch.int32, device=device)
    sums = torch.empty(K, d, dtype=torch.float64, device=device)
    cnt32 = torch.empty(K, dtype=torch.int32, device=device)
    offsets = torch.empty(K + 1, dtype=torch.int32, device=device)
    obj = torch.empty(1, dtype=torch.float64, device=device)

    def prepare(X):
        state["x"] = (X.data_ptr(), tuple(X.shape))
        state["split"] = fk.fk_split_points(X, out=planes) if planes is not None else None

    def assign(X, C):
        if planes is None:
            fk.fk_assign(X, C, labels, ws)
            return labels
        if state["x"] != (X.data_ptr(), tuple(X.shape)):
            raise ValueError("gpu_ops: prepare() was not called on these points")
        fk.fk_assign(state["split"], C, labels, ws)
        return labels

    def partial(X, lab, C):
        fk.fk_update_partial(X, lab, C, sums, cnt32, offsets, ws, objective=obj)
        return sums, cnt32.to(torch.int64), obj

    def finalize(sums_w, counts_w, objs_w, C_old):
        C_new = torch.empty_like(C_old)
        counts = torch.empty(C_old.shape[0], dtype=torch.int64, device=C_old.device)
        objective = torch.empty(1, dtype=torch.float64, device=C_old.device)
        fk.fk_finalize_shards(sums_w, counts_w, C_old, C_new, objectives_w=objs_w,
                              counts=counts, objective=objective)
        return C_new, counts, objective

    return LocalOps(assign, partial, finalize, prepare)


def _gather(t: torch.Tensor, world: int, group) -> torch.Tensor:
    """Stack every rank's copy of `t` along a new leading dimension, in rank order."""
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def lloyd_sharded(X_local: torch.Tensor, C: torch.Tensor, niter: int, ops: LocalOps,
                  group=None, timing: Optional[dict] = None):
    """Run `niter` data-parallel Lloyd iterations in place on C (replicated; every rank
    passes the same initial centroids).  Returns the list of global objectives (iteration
    t: sum over all ranks' points of ||x - c||^2 against the centroids of iteration t) and
    the global counts of the last iteration.

    With `timing` (a dict; CUDA tensors only) the device time of each phase is added to
    timing["ms_assign"], ["ms_partial"], ["ms_exchange"] and ["ms_finalize"], from CUDA
    events on the current stream (the stream the library calls run on)."""
    world = dist.get_world_size(group)
    objs = []
    counts = None
    ev = [] if timing is not None else None

    def mark():
        if ev is not None:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            ev.append(e)

    if ops.prepare is not None:
        ops.prepare(X_local)
    objective = None
    for _ in range(niter):
        mark()
        labels = ops.assign(X_local, C)
        mark()
        sums, cnt, obj = ops.partial(X_local, labels, C)
        mark()
        sums_w = _gather(sums, world, group)
        cnt_w = _gather(cnt, world, group)
        obj_w = _gather(obj.reshape(1), world, group).reshape(world)
        mark()
        C_new, counts, objective = ops.finalize(sums_w, cnt_w, obj_w, C)
        C.copy_(C_new)
        mark()
        objs.append(objective.reshape(-1)[:1].clone())
    objs = [float(o[0]) for o in objs]
    if ev:
        torch.cuda.current_stream().synchronize()
        names = ("ms_assign", "ms_partial", "ms_exchange", "ms_finalize")
        for t in range(niter):
            for p, name in enumerate(names):
                timing[name] = timing.get(name, 0.0) + ev[5 * t + p].elapsed_time(
                    ev[5 * t + p + 1])
    return objs, counts
