"""Expert parallelism over several GPUs: the host-side steps around ``mep_plan_rank``.

One process per GPU; each GPU is one expert-parallel rank holding its own S tokens
(R ranks in the process group). MoonEP places every token row straight at its final,
expert-grouped row on the destination rank (twodots.gr article on MoonEP, zero-copy
paragraph), so every rank must know the global balanced plan's rows for its own slots.
The plan orders slots by (e, src, t, k); the only information a rank lacks is how many
slots of each expert the other ranks hold. So the exchange step of the plan is one
all-gather of the R per-rank histograms (R x E int32), after which every rank derives
its rows and its exchange counts on its own GPU (``mep_plan_rank``); all ranks see the
same gathered matrix, so their shares form exactly the plan of ``mep_plan`` over the
ids of all ranks.

This module is plumbing only (the histogram and the plan run in the library's
kernels); its collectives go through ``torch.distributed`` (NCCL between GPUs).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _host_collectives(group) -> bool:
    """True when the group's backend moves host tensors only (gloo)."""
    return dist.get_backend(group) == "gloo"


def gather_histograms(hist: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of the ranks' per-expert histograms: int32 [R, E], row r = rank r's
    ``hist``, on ``hist``'s device. Every rank of ``group`` must call it with a
    histogram of the same length. Over gloo a device histogram goes through host memory."""
    if hist.dim() != 1 or hist.dtype != torch.int32:
        raise ValueError("hist must be a 1-D int32 tensor")
    world = dist.get_world_size(group)
    src = hist.contiguous()
    if src.is_cuda and _host_collectives(group):
        src = src.cpu()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    return torch.stack(parts).to(hist.device)


def share_buffers(buffers: dict, group=None) -> list:
    """Every rank's receive buffers, mapped into this process: CUDA IPC handles of this
    rank's tensors are all-gathered (as picklable objects over the process group) and the
    other ranks' handles opened here. Returns one dict per rank, ``buffers`` itself for
    this rank. The mapped tensors alias the other ranks' memory (on the same GPU, or on a
    peer GPU through NVLink); each rank must keep its own buffers alive, and the ranks
    must order their kernels on the buffers with a barrier, until every rank is done."""
    from torch.multiprocessing.reductions import reduce_tensor

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    mine = {k: reduce_tensor(v) for k, v in buffers.items()}
    every = [None] * world
    dist.all_gather_object(every, mine, group=group)
    out = []
    for r, handles in enumerate(every):
        if r == rank:
            out.append(buffers)
        else:
            out.append({k: fn(*args) for k, (fn, args) in handles.items()})
    return out


def plan_rank(ids: torch.Tensor, E: int, S: int, K: int, group=None, stream=None,
              out=None, histogram: Optional[Callable] = None, plan: Optional[Callable] = None):
    """This rank's share of the balanced plan: its per-expert histogram, the all-gather
    of every rank's histogram, then the rows of its S*K slots in the global plan and the
    counts of rows it sends to / receives from every rank.

    ``histogram(ids, E) -> int32 [E]`` and ``plan(ids, hist_all, R, E, S, K, rank, out)``
    default to the library's ``mep_histogram`` and ``mep_plan_rank``. Returns
    ``(out, hist_all)``; ``out`` holds pos, send_count, send_off, recv_count, recv_off.
    """
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if ids.numel() != S * K:
        raise ValueError("ids must hold this rank's S*K slots")
    if histogram is None or plan is None:
        import dispatch_combine_topk_b200 as mep
    if histogram is None:
        def histogram(i, n):
            h = torch.empty(n, dtype=torch.int32, device=i.device)
            return mep.mep_histogram(i, n, h, stream=stream)
    if plan is None:
        def plan(i, ha, R_, E_, S_, K_, r, o):
            o = o if o is not None else mep.RankPlanBuffers.allocate(R_, E_, S_, K_, i.device)
            return mep.mep_plan_rank(i, ha, R_, E_, S_, K_, r, o, stream=stream)
    hist = histogram(ids, E)
    if stream is not None and hist.is_cuda:
        # the collective waits for the histogram on the stream it was enqueued on
        with torch.cuda.stream(stream):
            hist_all = gather_histograms(hist, group)
    else:
        hist_all = gather_histograms(hist, group)
    return plan(ids, hist_all, R, E, S, K, rank, out), hist_all
