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

The exchange itself is one kernel per direction: every rank dispatches its own token
rows straight into the receive buffers of all ranks (peer stores through a table of their
addresses, ``mep_dispatch_ranks``), and combines its tokens by reading the expert outputs
from all ranks' buffers (``mep_combine_ranks``). ``Exchange`` holds one rank's side:
its buffer, shared with the group through CUDA IPC, and the address tables. The ranks
meet only in host barriers between the phases; no kernel waits on another process.

This module is plumbing only (the histogram, the plan and the exchange run in the
library's kernels); its collectives go through ``torch.distributed`` (NCCL between GPUs).
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


class Exchange:
    """One EP rank's side of the token exchange over a process group of R ranks, each
    holding S tokens of K slots and an [S*K, H] receive buffer (bf16, or int8 codes with
    fp32 scales for ``quant=1``).

    Construction is collective: every rank allocates its buffer and maps every other
    rank's (``share_buffers``). Per step:

    - ``plan(ids)``: this rank's rows in the global plan (``plan_rank``);
    - ``dispatch(x, rp)``: its token rows into every rank's buffer (peer stores);
    - ``fence()``: waits for this rank's stream, then for every rank (host barrier), so
      that the rows written by all ranks are in place before anyone reads them; call it
      after ``dispatch``, after the experts have written their outputs into ``rows``,
      and after ``combine`` before the next ``dispatch`` overwrites the buffers;
    - ``combine(rp, gates, out)``: its tokens' gate-weighted sum read from every rank's
      buffer.

    ``close()`` (collective) ends the sharing: no rank frees its buffer while another
    may still read it."""

    def __init__(self, E: int, S: int, K: int, H: int, quant: int = 0, group=None, device=None, stream=None):
        import dispatch_combine_topk_b200 as mep
        self._mep = mep
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.S, self.K, self.H, self.quant = E, S, K, H, quant
        self.rows_per_rank = S * K
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.stream = stream
        dt = torch.int8 if quant else torch.bfloat16
        self.rows = torch.zeros((self.rows_per_rank, H), dtype=dt, device=self.device)
        mine = {"rows": self.rows}
        self.scale = None
        if quant:
            self.scale = torch.zeros(self.rows_per_rank, dtype=torch.float32, device=self.device)
            mine["scale"] = self.scale
        torch.cuda.synchronize(self.device)              # the buffers exist before they are shared
        self._every = share_buffers(mine, group)
        self.table = mep.rank_pointer_table([b["rows"] for b in self._every], self.device)
        self.scale_table = (mep.rank_pointer_table([b["scale"] for b in self._every], self.device)
                            if quant else None)

    def plan(self, ids: torch.Tensor, out=None):
        """This rank's rows in the global plan and its exchange counts (``plan_rank``).
        Returns ``(RankPlanBuffers, hist_all)``."""
        return plan_rank(ids, self.E, self.S, self.K, self.group, stream=self.stream, out=out)

    def dispatch(self, x: torch.Tensor, rp) -> None:
        """This rank's token rows x [S, H] into every rank's buffer, at the rows ``rp.pos``."""
        self._mep.mep_dispatch_ranks(x, rp.pos, self.K, self.table, self.rows_per_rank, quant=self.quant,
                                     scale_table=self.scale_table, stream=self.stream)

    def fence(self) -> None:
        """This rank's work on its stream done, then every rank's (host barrier)."""
        if self.stream is not None:
            self.stream.synchronize()
        else:
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)

    def combine(self, rp, gates: torch.Tensor, out: torch.Tensor) -> torch.Tensor:
        """out [S, H] (bf16) = the gate-weighted sum of this rank's slots, read from the
        buffers of the ranks they went to."""
        self._mep.mep_combine_ranks(self.table, rp.pos, gates, self.K, self.rows_per_rank, out, quant=self.quant,
                                    scale_table=self.scale_table, stream=self.stream)
        return out

    def close(self) -> None:
        """Collective: every rank stops reading the others' buffers, then drops them."""
        self.fence()
        self._every = None
        self.table = self.scale_table = None
