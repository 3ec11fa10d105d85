"""MoE expert-parallel token routing on one B200: Python binding of libmep.

Every function here is argument marshalling around the C ABI declared in
``include/mep.h`` (same names): it checks dtypes and devices of torch tensors, passes
their device pointers and the current CUDA stream, and raises ``MepError`` on a
non-OK status. All computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback. If ``libmep.so`` has not been built, importing the binding's
functions raises immediately.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmep.so")

MEP_PLAN_BALANCED = 0
MEP_PLAN_GROUPED = 1
MEP_MAX_KEYS = 4096
MEP_MAX_K = 32

DERR_KEY_RANGE = 0x1
DERR_ROW_RANGE = 0x2
DERR_TABLE = 0x4
DERR_MASK = 0x8
DERR_TIMEOUT = 0x10
DERR_DRAIN = 0x20
DERR_HIST = 0x40

STATUS = {0: "MEP_OK", 1: "MEP_ERR_NULLPTR", 2: "MEP_ERR_DTYPE", 3: "MEP_ERR_SHAPE",
          4: "MEP_ERR_VALUE", 5: "MEP_ERR_WORKSPACE", 6: "MEP_ERR_CUDA", 7: "MEP_ERR_TIMEOUT"}


class MepError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = STATUS.get(status, str(status))
        extra = ""
        if status == 6:
            extra = f" (cudaError {lib().mep_last_cuda_error()})"
        super().__init__(f"{what}: {name}{extra}")


class _RouteBuffersC(ctypes.Structure):
    """mep_route_buffers_t of include/mep.h."""
    _fields_ = [("R", ctypes.c_int32), ("E", ctypes.c_int32), ("S", ctypes.c_int32), ("K", ctypes.c_int32),
                ("H", ctypes.c_int64), ("quant", ctypes.c_int32)] + \
               [(n, ctypes.c_void_p) for n in ("ids", "gates", "x", "recv", "recv_scale", "out", "pos", "hist",
                                               "rank_off", "load", "rep_count", "rep_key", "rep_cu", "stats",
                                               "workspace")] + \
               [("workspace_bytes", ctypes.c_size_t)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmep.so (built in-tree by ``dispatch_combine_topk_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmep.so not found at {LIB_PATH}; build it with "
                              "`python -m dispatch_combine_topk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.mep_version.restype = i32
        L.mep_status_string.argtypes = [ctypes.c_int]
        L.mep_status_string.restype = ctypes.c_char_p
        L.mep_last_cuda_error.restype = i32
        L.mep_get_error.argtypes = [P, P, i32]
        L.mep_histogram.argtypes = [P, i64, i32, P, P]
        L.mep_plan_workspace_size.argtypes = [i32, i32, i32, i32]
        L.mep_plan_workspace_size.restype = ctypes.c_size_t
        L.mep_plan_launches.argtypes = [i32, i32, i32, i32]
        L.mep_plan_launches.restype = i32
        L.mep_plan.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P,
                               ctypes.c_size_t, P]
        L.mep_update_expert.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i64, i64, P, P, P]
        L.mep_dispatch.argtypes = [P, P, i64, i32, i64, i32, P, P, i64, P]
        L.mep_dequantize.argtypes = [P, P, i64, i64, P, P]
        L.mep_combine.argtypes = [P, i64, P, P, i64, i32, i64, P, P]
        L.mep_combine_int8.argtypes = [P, P, i64, P, P, i64, i32, i64, P, P]
        L.mep_combine_add_rmsnorm.argtypes = [P, i64, P, P, i64, i32, i64, P, P, ctypes.c_float,
                                              P, P, P, P]
        L.mep_prefetch_plan.argtypes = [P, P, i32, i32, i32, i32, P, P, P]
        L.mep_prefetch_weights.argtypes = [P, P, i32, i32, i32, i64, P, P]
        L.mep_grad_reduce.argtypes = [P, P, P, i32, i32, i32, i64, P]
        L.mep_dispatch_int8_smooth.argtypes = [P, P, P, i64, i32, i64, P, i32, P, P, i64, P]
        L.mep_update_expert_ranks.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i64, P, P, P]
        L.mep_dispatch_int8_smooth_workspace_size.argtypes = [i64, i32]
        L.mep_dispatch_int8_smooth_workspace_size.restype = ctypes.c_size_t
        L.mep_dispatch_int8_smooth_grouped.argtypes = [P, P, P, i64, i32, i64, P, i32, P, P, i64, P,
                                                       ctypes.c_size_t, P]
        L.mep_dedup_workspace_size.argtypes = [i32, i32, i32]
        L.mep_dedup_workspace_size.restype = ctypes.c_size_t
        L.mep_dedup_plan.argtypes = [P, P, i32, i32, i32, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.mep_expand.argtypes = [P, P, i64, P, i64, i64, i32, P, P, P]
        L.mep_route_host.argtypes = [ctypes.POINTER(_RouteBuffersC), P, P, P, P, P]
        L.mep_stream_synchronize_timeout.argtypes = [P, i32]
        L.mep_maxvio.argtypes = [P, i32, i32, i32, P, P, P]
        L.mep_plan_rank_workspace_size.argtypes = [i32, i32, i32, i32]
        L.mep_plan_rank_workspace_size.restype = ctypes.c_size_t
        L.mep_plan_rank.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.mep_plan_static_ws.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]
        L.mep_dispatch_ranks.argtypes = [P, P, i64, i32, i64, i32, P, P, i32, i64, P]
        L.mep_combine_ranks.argtypes = [P, P, i32, i32, i64, P, P, i64, i32, i64, P, P]
        for f in ["mep_get_error", "mep_histogram", "mep_plan", "mep_update_expert",
                  "mep_dispatch", "mep_dequantize", "mep_combine", "mep_combine_int8",
                  "mep_combine_add_rmsnorm", "mep_prefetch_plan", "mep_prefetch_weights",
                  "mep_grad_reduce", "mep_dispatch_int8_smooth", "mep_dispatch_int8_smooth_grouped",
                  "mep_update_expert_ranks",
                  "mep_dedup_plan", "mep_expand", "mep_route_host", "mep_stream_synchronize_timeout",
                  "mep_maxvio", "mep_plan_rank", "mep_plan_static_ws", "mep_dispatch_ranks",
                  "mep_combine_ranks"]:
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _need(ok: bool, what: str):
    """Shape check of the binding: the C calls cannot see the sizes of device buffers,
    so a tensor too small for the call is refused here, before anything is launched."""
    if not ok:
        raise ValueError(what)


def _n(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel()


def _check_plan_buffers(out: "PlanBuffers", R: int, n_keys: int, N: int):
    _need(_n(out.pos) >= N and _n(out.hist) >= n_keys and _n(out.rank_off) >= R + 1
          and (out.load is None or _n(out.load) >= R) and _n(out.rep_count) >= R
          and _n(out.rep_key) >= R * n_keys and _n(out.rep_cu) >= R * (n_keys + 1) and _n(out.stats) >= 8,
          "plan buffers too small for (R, n_keys, S, K): allocate them with PlanBuffers.allocate")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ok(rc: int, what: str):
    if rc != 0:
        raise MepError(rc, what)


def mep_get_error(clear: bool = True, stream=None) -> int:
    """Sticky error word of the current device, read in order on `stream` (default: the
    current stream); waits for that stream only. With clear, the bits read are cleared."""
    code = ctypes.c_int32(0)
    _ok(lib().mep_get_error(_stream(stream), ctypes.byref(code), int(clear)), "mep_get_error")
    return code.value


def mep_stream_synchronize_timeout(timeout_ms: int, stream=None) -> bool:
    """Wait for the stream's work for at most timeout_ms: True when it finished, False
    on time-out (the work keeps running). Raises MepError on a CUDA error."""
    rc = lib().mep_stream_synchronize_timeout(_stream(stream), int(timeout_ms))
    if rc == 7:
        return False
    _ok(rc, "mep_stream_synchronize_timeout")
    return True


def mep_histogram(ids: torch.Tensor, n_keys: int, hist: torch.Tensor, stream=None):
    """hist[e] = slots of ids equal to e (int32 [n_keys]); ids int32, any length."""
    _need(_n(hist) >= n_keys, "hist must hold n_keys counts")
    _ok(lib().mep_histogram(_ptr(ids, torch.int32, "ids"), ids.numel(), n_keys,
                            _ptr(hist, torch.int32, "hist"), _stream(stream)), "mep_histogram")
    return hist


def mep_plan_workspace_size(R: int, n_keys: int, S: int, K: int) -> int:
    """Bytes of scratch mep_plan needs for this shape (PlanBuffers.allocate uses it)."""
    return int(lib().mep_plan_workspace_size(R, n_keys, S, K))


def mep_plan_launches(R: int, n_keys: int, S: int, K: int) -> int:
    """Kernels mep_plan launches for this shape (1: one launch; 3: the tiled sort)."""
    return int(lib().mep_plan_launches(R, n_keys, S, K))


@dataclasses.dataclass
class PlanBuffers:
    """Device outputs of mep_plan (see include/mep.h for their layout)."""

    pos: torch.Tensor        # int32 [N]
    hist: torch.Tensor       # int32 [n_keys]
    rank_off: torch.Tensor   # int32 [R+1]
    load: torch.Tensor       # int32 [R]
    rep_count: torch.Tensor  # int32 [R]
    rep_key: torch.Tensor    # int32 [R, n_keys]
    rep_cu: torch.Tensor     # int32 [R, n_keys+1]
    stats: torch.Tensor      # int32 [8] (mep_plan_stats_t)
    workspace: torch.Tensor  # uint8, 256-byte aligned

    @staticmethod
    def allocate(R: int, n_keys: int, S: int, K: int, device=None) -> "PlanBuffers":
        dev = device or torch.device("cuda", torch.cuda.current_device())
        z = lambda *s: torch.empty(s, dtype=torch.int32, device=dev)
        ws = torch.empty(max(256, mep_plan_workspace_size(R, n_keys, S, K)), dtype=torch.uint8,
                         device=dev)
        return PlanBuffers(z(R * S * K), z(n_keys), z(R + 1), z(R), z(R), z(R, n_keys),
                           z(R, n_keys + 1), z(8), ws)

    def stats_dict(self) -> dict:
        s = self.stats.tolist()
        return dict(max_load=s[0], max_chunk=s[1], redundant=s[2], prefetched=s[3], n_kept=s[4],
                    max_hist=s[5], n_ranks_used=s[6])


def mep_plan(ids: torch.Tensor, R: int, n_keys: int, S: int, K: int, out: PlanBuffers,
             mode: int = MEP_PLAN_BALANCED, keys_per_rank: int = 0,
             keep: Optional[torch.Tensor] = None, stream=None) -> PlanBuffers:
    """The placement plan of R*S*K slots (balanced: every rank exactly S*K rows; grouped:
    by physical instance with dropped slots) into `out` (see include/mep.h)."""
    if ids.numel() != R * S * K:
        raise ValueError("ids must hold R*S*K slots")
    _need(keep is None or keep.numel() == R * S * K, "keep must hold R*S*K flags")
    _check_plan_buffers(out, R, n_keys, R * S * K)
    rc = lib().mep_plan(_ptr(ids, torch.int32, "ids"), _ptr(keep, torch.uint8, "keep"), R, n_keys,
                        S, K, mode, keys_per_rank, _ptr(out.pos), _ptr(out.hist),
                        _ptr(out.rank_off), _ptr(out.load), _ptr(out.rep_count),
                        _ptr(out.rep_key), _ptr(out.rep_cu), _ptr(out.stats),
                        _ptr(out.workspace), out.workspace.numel(), _stream(stream))
    _ok(rc, "mep_plan")
    return out


def mep_maxvio(stats, S: int, K: int, n_keys: int) -> dict:
    """maxvio before and after the plan, and over experts, from a plan summary (the
    PlanBuffers' stats tensor on any device, or 8 ints); host arithmetic only."""
    vals = (stats.tolist() if hasattr(stats, "tolist") else list(stats))[:8]
    buf = (ctypes.c_int32 * 8)(*[int(v) for v in vals])
    out = [ctypes.c_double(0.0) for _ in range(3)]
    _ok(lib().mep_maxvio(ctypes.cast(buf, ctypes.c_void_p), S, K, n_keys, *[ctypes.byref(o) for o in out]),
        "mep_maxvio")
    return {"rank_before": out[0].value, "rank_after": out[1].value, "expert": out[2].value}


def mep_plan_rank_workspace_size(R: int, E: int, S: int, K: int) -> int:
    """Bytes of scratch mep_plan_rank needs for this shape."""
    return int(lib().mep_plan_rank_workspace_size(R, E, S, K))


@dataclasses.dataclass
class RankPlanBuffers:
    """Device outputs of mep_plan_rank: one EP rank's share of the balanced plan."""

    pos: torch.Tensor         # int32 [S*K]: global row of each of this rank's slots
    send_count: torch.Tensor  # int32 [R]
    send_off: torch.Tensor    # int32 [R+1]
    recv_count: torch.Tensor  # int32 [R]
    recv_off: torch.Tensor    # int32 [R+1]
    workspace: torch.Tensor   # uint8, 256-byte aligned

    @staticmethod
    def allocate(R: int, E: int, S: int, K: int, device=None) -> "RankPlanBuffers":
        dev = device or torch.device("cuda", torch.cuda.current_device())
        z = lambda n: torch.empty(n, dtype=torch.int32, device=dev)
        ws = torch.empty(max(256, mep_plan_rank_workspace_size(R, E, S, K)), dtype=torch.uint8, device=dev)
        return RankPlanBuffers(z(S * K), z(R), z(R + 1), z(R), z(R + 1), ws)


def mep_plan_rank(ids: torch.Tensor, hist_all: torch.Tensor, R: int, E: int, S: int, K: int, rank: int,
                  out: RankPlanBuffers, stream=None) -> RankPlanBuffers:
    """Rank `rank`'s share of the balanced plan from the all-gathered per-rank histograms
    hist_all (int32 [R, E]): the global rows of its S*K slots and the exchange counts."""
    _need(ids.numel() == S * K, "ids must hold this rank's S*K slots")
    _need(hist_all.numel() == R * E, "hist_all must be [R, E]")
    _need(_n(out.pos) >= S * K and _n(out.send_count) >= R and _n(out.send_off) >= R + 1
          and _n(out.recv_count) >= R and _n(out.recv_off) >= R + 1,
          "rank plan buffers too small: allocate them with RankPlanBuffers.allocate")
    rc = lib().mep_plan_rank(_ptr(ids, torch.int32, "ids"), _ptr(hist_all, torch.int32, "hist_all"), R, E, S, K,
                             rank, _ptr(out.pos, torch.int32), _ptr(out.send_count, torch.int32),
                             _ptr(out.send_off, torch.int32), _ptr(out.recv_count, torch.int32),
                             _ptr(out.recv_off, torch.int32), _ptr(out.workspace), out.workspace.numel(),
                             _stream(stream))
    _ok(rc, "mep_plan_rank")
    return out


def rank_pointer_table(buffers, device=None) -> torch.Tensor:
    """A device array of the ranks' buffer addresses (int64 [R]) for mep_dispatch_ranks /
    mep_combine_ranks: one tensor per rank, on this device or (across GPUs) a peer
    mapping of another GPU's buffer."""
    dev = device or buffers[0].device
    return torch.tensor([b.data_ptr() for b in buffers], dtype=torch.int64).to(dev)


def mep_dispatch_ranks(x: torch.Tensor, pos: torch.Tensor, K: int, recv_table: torch.Tensor, rows_per_rank: int,
                       quant: int = 0, scale_table: Optional[torch.Tensor] = None, stream=None):
    """Dispatch into the ranks' own buffers (see include/mep.h): slot n's row goes to
    rank pos[n] // rows_per_rank at local row pos[n] % rows_per_rank, through a device
    table of buffer addresses (rank_pointer_table)."""
    T, H = x.shape
    _need(pos.numel() == T * K, "pos must hold T*K slots")
    _need(recv_table.dtype == torch.int64 and recv_table.dim() == 1, "recv_table: int64 [R] addresses")
    R = recv_table.numel()
    _need(quant == 0 or (scale_table is not None and scale_table.numel() == R), "scale_table [R] needed for int8")
    _ok(lib().mep_dispatch_ranks(_ptr(x, torch.bfloat16, "x"), _ptr(pos, torch.int32, "pos"), T, K, H, quant,
                                 _ptr(recv_table, torch.int64, "recv_table"),
                                 _ptr(scale_table, torch.int64, "scale_table"), R, rows_per_rank, _stream(stream)),
        "mep_dispatch_ranks")


def mep_combine_ranks(y_table: torch.Tensor, pos: torch.Tensor, gates: torch.Tensor, K: int, rows_per_rank: int,
                      out: torch.Tensor, quant: int = 0, scale_table: Optional[torch.Tensor] = None, stream=None):
    """Combine from the ranks' own buffers (see include/mep.h)."""
    T, H = out.shape
    _need(pos.numel() == T * K and gates.numel() == T * K, "pos and gates must hold T*K slots")
    _need(y_table.dtype == torch.int64 and y_table.dim() == 1, "y_table: int64 [R] addresses")
    R = y_table.numel()
    _need(quant == 0 or (scale_table is not None and scale_table.numel() == R), "scale_table [R] needed for int8")
    _ok(lib().mep_combine_ranks(_ptr(y_table, torch.int64, "y_table"), _ptr(scale_table, torch.int64, "scale_table"),
                                quant, R, rows_per_rank, _ptr(pos, torch.int32, "pos"),
                                _ptr(gates, torch.float32, "gates"), T, K, H, _ptr(out, torch.bfloat16, "out"),
                                _stream(stream)),
        "mep_combine_ranks")
    return out


def mep_dedup_workspace_size(R: int, S: int, K: int) -> int:
    """Bytes of scratch mep_dedup_plan needs (DedupBuffers.allocate uses it)."""
    return int(lib().mep_dedup_workspace_size(R, S, K))


@dataclasses.dataclass
class DedupBuffers:
    """Device outputs of mep_dedup_plan: one row per (token, destination rank)."""

    dsend: torch.Tensor      # int32 [N]  row of each pair's first slot (the send list), else -1
    dpos: torch.Tensor       # int32 [N]  row of every kept slot
    drank_off: torch.Tensor  # int32 [R+1]
    dtok: torch.Tensor       # int32 [N]  token of every row, -1 past drank_off[R]
    gidx: torch.Tensor       # int32 [N]  row holding the token of every plan row
    workspace: torch.Tensor  # uint8, 256-byte aligned

    @staticmethod
    def allocate(R: int, S: int, K: int, device=None) -> "DedupBuffers":
        dev = device or torch.device("cuda", torch.cuda.current_device())
        N = R * S * K
        z = lambda n: torch.empty(n, dtype=torch.int32, device=dev)
        ws = torch.empty(max(256, mep_dedup_workspace_size(R, S, K)), dtype=torch.uint8, device=dev)
        return DedupBuffers(z(N), z(N), z(R + 1), z(N), z(N), ws)


def mep_dedup_plan(pos: torch.Tensor, rank_off: torch.Tensor, R: int, S: int, K: int, out: DedupBuffers,
                   stream=None) -> DedupBuffers:
    """One row per (token, destination rank) from a plan's pos and rank_off: the send
    list, every slot's row, the ranks' first rows, each row's token and the plan rows'
    source rows (see include/mep.h)."""
    if pos.numel() != R * S * K or rank_off.numel() != R + 1:
        raise ValueError("pos must hold R*S*K slots and rank_off R+1 offsets")
    N = R * S * K
    _need(min(_n(out.dsend), _n(out.dpos), _n(out.dtok), _n(out.gidx)) >= N and _n(out.drank_off) >= R + 1,
          "dedup buffers too small: allocate them with DedupBuffers.allocate")
    rc = lib().mep_dedup_plan(_ptr(pos, torch.int32, "pos"), _ptr(rank_off, torch.int32, "rank_off"), R, S, K,
                              _ptr(out.dsend), _ptr(out.dpos), _ptr(out.drank_off), _ptr(out.dtok),
                              _ptr(out.gidx), _ptr(out.workspace), out.workspace.numel(), _stream(stream))
    _ok(rc, "mep_dedup_plan")
    return out


def mep_expand(src: torch.Tensor, gidx: torch.Tensor, dst: torch.Tensor, src_scale: Optional[torch.Tensor] = None,
               dst_scale: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dst[p] = src[gidx[p]] for gidx[p] >= 0: bf16 rows, or int8 rows with their scales."""
    quant = 1 if src.dtype == torch.int8 else 0
    want = torch.int8 if quant else torch.bfloat16
    rows, H = dst.shape
    if src.dim() != 2 or src.shape[1] != H or gidx.numel() != rows:
        raise ValueError("src [rows_src, H], dst [rows, H] and gidx [rows] must agree")
    _need(dst.dtype == src.dtype, "src and dst must have the same dtype")
    if quant:
        _need(_n(src_scale) >= src.shape[0] and _n(dst_scale) >= rows, "int8 rows need src and dst scales")
    rc = lib().mep_expand(_ptr(src, want, "src"), _ptr(src_scale, torch.float32, "src_scale"), src.shape[0],
                          _ptr(gidx, torch.int32, "gidx"), rows, H, quant, _ptr(dst, want, "dst"),
                          _ptr(dst_scale, torch.float32, "dst_scale"), _stream(stream))
    _ok(rc, "mep_expand")
    return dst


def _check_mapping(ids, scales, thr, active, out_ids, out_mask):
    rows, K = ids.shape
    _need(scales is None or tuple(scales.shape) == (rows, K), "expert_scales must match expert_ids")
    _need(thr is None or thr.numel() == K, "pruning_threshold must hold K values")
    _need(active is None or active.numel() == rows, "active_mask must hold one flag per token")
    _need(_n(out_ids) >= rows * K and _n(out_mask) >= rows * K, "outputs must hold one entry per slot")


def mep_update_expert(expert_ids: torch.Tensor, eplb_table: torch.Tensor,
                      expert_scales: Optional[torch.Tensor], pruning_threshold: Optional[torch.Tensor],
                      active_mask: Optional[torch.Tensor], local_rank_id: int, world_size: int,
                      balance_mode: int, balanced_expert_ids: torch.Tensor,
                      balanced_active_mask: torch.Tensor, stream=None):
    """Logical -> physical expert ids through eplb_table (balance_mode 0 by rank, 1 by
    token) and the pruning mask, for one rank's BS tokens."""
    BS, K = expert_ids.shape
    E, F = eplb_table.shape
    _check_mapping(expert_ids, expert_scales, pruning_threshold, active_mask, balanced_expert_ids,
                   balanced_active_mask)
    rc = lib().mep_update_expert(_ptr(expert_ids, torch.int32, "expert_ids"),
                                 _ptr(eplb_table, torch.int32, "eplb_table"),
                                 _ptr(expert_scales, torch.float32, "expert_scales"),
                                 _ptr(pruning_threshold, torch.float32, "pruning_threshold"),
                                 _ptr(active_mask, torch.uint8, "active_mask"), BS, K, E, F,
                                 local_rank_id, world_size, balance_mode,
                                 _ptr(balanced_expert_ids, torch.int32, "balanced_expert_ids"),
                                 _ptr(balanced_active_mask, torch.uint8, "balanced_active_mask"),
                                 _stream(stream))
    _ok(rc, "mep_update_expert")
    return balanced_expert_ids, balanced_active_mask


def mep_update_expert_ranks(expert_ids: torch.Tensor, eplb_table: torch.Tensor,
                            expert_scales: Optional[torch.Tensor],
                            pruning_threshold: Optional[torch.Tensor],
                            active_mask: Optional[torch.Tensor], world_size: int, balance_mode: int,
                            balanced_expert_ids: torch.Tensor, balanced_active_mask: torch.Tensor,
                            stream=None):
    """mep_update_expert for every simulated rank in one launch (rows = world_size blocks)."""
    rows, K = expert_ids.shape
    E, F = eplb_table.shape
    _need(world_size >= 1 and rows % world_size == 0, "expert_ids must hold world_size blocks of BS tokens")
    _check_mapping(expert_ids, expert_scales, pruning_threshold, active_mask, balanced_expert_ids,
                   balanced_active_mask)
    rc = lib().mep_update_expert_ranks(_ptr(expert_ids, torch.int32, "expert_ids"),
                                       _ptr(eplb_table, torch.int32, "eplb_table"),
                                       _ptr(expert_scales, torch.float32, "expert_scales"),
                                       _ptr(pruning_threshold, torch.float32, "pruning_threshold"),
                                       _ptr(active_mask, torch.uint8, "active_mask"), rows // world_size,
                                       K, E, F, world_size, balance_mode,
                                       _ptr(balanced_expert_ids, torch.int32, "balanced_expert_ids"),
                                       _ptr(balanced_active_mask, torch.uint8, "balanced_active_mask"),
                                       _stream(stream))
    _ok(rc, "mep_update_expert_ranks")
    return balanced_expert_ids, balanced_active_mask


def mep_dispatch(x: torch.Tensor, pos: torch.Tensor, K: int, recv: torch.Tensor,
                 recv_scale: Optional[torch.Tensor] = None, quant: int = 0, stream=None):
    """recv[pos[n]] = x[n // K] for every kept slot (bf16), or its per-token int8 codes
    with the scale in recv_scale (quant=1). x bf16 [T, H], pos int32 [T*K], recv [rows, H]."""
    T, H = x.shape
    want = torch.int8 if quant == 1 else torch.bfloat16
    rows = recv.shape[0]
    _need(pos.numel() == T * K, "pos must hold T*K slots")
    _need(recv.dim() == 2 and recv.shape[1] == H, "recv must be [rows, H]")
    _need(quant != 1 or _n(recv_scale) >= rows, "int8 dispatch needs recv_scale [rows]")
    rc = lib().mep_dispatch(_ptr(x, torch.bfloat16, "x"), _ptr(pos, torch.int32, "pos"), T, K, H,
                            quant, _ptr(recv, want, "recv"),
                            _ptr(recv_scale, torch.float32, "recv_scale"), rows, _stream(stream))
    _ok(rc, "mep_dispatch")
    return recv


def mep_dequantize(q: torch.Tensor, scale: torch.Tensor, y: torch.Tensor, stream=None):
    """y = bf16(q * scale) row by row: the identity expert on int8 rows."""
    rows, H = q.shape
    _need(_n(scale) >= rows and tuple(y.shape) == (rows, H), "scale [rows] and y [rows, H] must match q")
    _ok(lib().mep_dequantize(_ptr(q, torch.int8, "q"), _ptr(scale, torch.float32, "scale"), rows, H,
                             _ptr(y, torch.bfloat16, "y"), _stream(stream)), "mep_dequantize")
    return y


def _check_combine(y, pos, gates, T, K, H):
    _need(y.dim() == 2 and y.shape[1] == H, "y must be [rows, H] with out's H")
    _need(pos.numel() == T * K and gates.numel() == T * K, "pos and gates must hold T*K slots")


def mep_combine(y: torch.Tensor, pos: torch.Tensor, gates: torch.Tensor, K: int,
                out: torch.Tensor, stream=None):
    """out[t] = bf16(sum over kept k, ascending, of fl(gate * y[pos[t*K+k]])) in fp32.
    y bf16 [rows, H], pos int32 [T*K], gates fp32 [T*K], out bf16 [T, H]."""
    T, H = out.shape
    _check_combine(y, pos, gates, T, K, H)
    rc = lib().mep_combine(_ptr(y, torch.bfloat16, "y"), y.shape[0], _ptr(pos, torch.int32, "pos"),
                           _ptr(gates, torch.float32, "gates"), T, K, H,
                           _ptr(out, torch.bfloat16, "out"), _stream(stream))
    _ok(rc, "mep_combine")
    return out


def mep_combine_int8(yq: torch.Tensor, y_scale: torch.Tensor, pos: torch.Tensor, gates: torch.Tensor,
                     K: int, out: torch.Tensor, stream=None):
    """Combine of int8 rows with per-row scales (dequantisation fused into the sum)."""
    T, H = out.shape
    _check_combine(yq, pos, gates, T, K, H)
    _need(_n(y_scale) >= yq.shape[0], "y_scale must hold one scale per row")
    rc = lib().mep_combine_int8(_ptr(yq, torch.int8, "yq"), _ptr(y_scale, torch.float32, "y_scale"),
                                yq.shape[0], _ptr(pos, torch.int32, "pos"),
                                _ptr(gates, torch.float32, "gates"), T, K, H,
                                _ptr(out, torch.bfloat16, "out"), _stream(stream))
    _ok(rc, "mep_combine_int8")
    return out


def mep_combine_add_rmsnorm(y: torch.Tensor, pos: torch.Tensor, gates: torch.Tensor, K: int,
                            residual: torch.Tensor, gamma: torch.Tensor, eps: float,
                            x_out: torch.Tensor, y_out: torch.Tensor, rstd_out: torch.Tensor,
                            stream=None):
    """Combine, residual add and RMSNorm in one kernel (see include/mep.h)."""
    T, H = x_out.shape
    _check_combine(y, pos, gates, T, K, H)
    _need(tuple(residual.shape) == (T, H) and tuple(y_out.shape) == (T, H) and gamma.numel() == H
          and _n(rstd_out) >= T, "residual, y_out [T, H], gamma [H] and rstd_out [T] must match")
    rc = lib().mep_combine_add_rmsnorm(
        _ptr(y, torch.bfloat16, "y"), y.shape[0], _ptr(pos, torch.int32, "pos"),
        _ptr(gates, torch.float32, "gates"), T, K, H, _ptr(residual, torch.bfloat16, "residual"),
        _ptr(gamma, torch.bfloat16, "gamma"), float(eps), _ptr(x_out, torch.bfloat16, "x_out"),
        _ptr(y_out, torch.bfloat16, "y_out"), _ptr(rstd_out, torch.float32, "rstd_out"),
        _stream(stream))
    _ok(rc, "mep_combine_add_rmsnorm")
    return x_out, y_out, rstd_out


def mep_prefetch_plan(plan: PlanBuffers, R: int, E: int, B: int, slot_expert: torch.Tensor,
                      rep_weight: torch.Tensor, stream=None):
    """Slots of the prefetched replicas and the weight row of every replica."""
    cap = plan.rep_key.shape[1]
    _need(plan.rep_key.shape[0] >= R and _n(plan.rep_count) >= R, "plan buffers must cover R ranks")
    _need(B == 0 or _n(slot_expert) >= R * B, "slot_expert must hold R*B slots")
    _need(_n(rep_weight) >= R * cap, "rep_weight must be [R, cap]")
    rc = lib().mep_prefetch_plan(_ptr(plan.rep_count, torch.int32, "rep_count"),
                                 _ptr(plan.rep_key, torch.int32, "rep_key"), R, E, cap, B,
                                 _ptr(slot_expert, torch.int32, "slot_expert") if B > 0 else None,
                                 _ptr(rep_weight, torch.int32, "rep_weight"), _stream(stream))
    _ok(rc, "mep_prefetch_plan")
    return slot_expert, rep_weight


def mep_prefetch_weights(w_home: torch.Tensor, slot_expert: torch.Tensor, R: int, B: int,
                         w_slots: torch.Tensor, stream=None):
    """w_slots[s] = w_home[slot_expert[s]] for every used slot (bf16 expert weights)."""
    E = w_home.shape[0]
    D = w_home.numel() // E
    _need(_n(slot_expert) >= R * B and _n(w_slots) >= R * B * D, "slot_expert [R*B] and w_slots [R*B, ...] needed")
    rc = lib().mep_prefetch_weights(_ptr(w_home, torch.bfloat16, "w_home"),
                                    _ptr(slot_expert, torch.int32, "slot_expert"), E, R, B, D,
                                    _ptr(w_slots, torch.bfloat16, "w_slots"), _stream(stream))
    _ok(rc, "mep_prefetch_weights")
    return w_slots


def mep_grad_reduce(grad_home: torch.Tensor, grad_slots: torch.Tensor, slot_expert: torch.Tensor,
                    R: int, B: int, stream=None):
    """grad_home[e] += its slots in ascending (rank, slot) order (fp32), then the slots
    are cleared."""
    E = grad_home.shape[0]
    D = grad_home.numel() // E
    _need(_n(slot_expert) >= R * B and _n(grad_slots) >= R * B * D,
          "slot_expert [R*B] and grad_slots [R*B, ...] needed")
    rc = lib().mep_grad_reduce(_ptr(grad_home, torch.float32, "grad_home"),
                               _ptr(grad_slots, torch.float32, "grad_slots"),
                               _ptr(slot_expert, torch.int32, "slot_expert"), E, R, B, D,
                               _stream(stream))
    _ok(rc, "mep_grad_reduce")
    return grad_home, grad_slots


def mep_dispatch_int8_smooth(x: torch.Tensor, ids: torch.Tensor, pos: torch.Tensor, K: int,
                             smooth: torch.Tensor, recv: torch.Tensor, recv_scale: torch.Tensor,
                             stream=None):
    """int8 dispatch with per-expert smoothing scales (codes and scale per slot)."""
    T, H = x.shape
    _need(ids.numel() == T * K and pos.numel() == T * K, "ids and pos must hold T*K slots")
    _need(smooth.dim() == 2 and smooth.shape[1] == H, "smooth must be [experts, H]")
    _need(recv.dim() == 2 and recv.shape[1] == H and _n(recv_scale) >= recv.shape[0],
          "recv [rows, H] and recv_scale [rows] needed")
    rc = lib().mep_dispatch_int8_smooth(_ptr(x, torch.bfloat16, "x"), _ptr(ids, torch.int32, "ids"),
                                        _ptr(pos, torch.int32, "pos"), T, K, H,
                                        _ptr(smooth, torch.float32, "smooth"), smooth.shape[0],
                                        _ptr(recv, torch.int8, "recv"),
                                        _ptr(recv_scale, torch.float32, "recv_scale"), recv.shape[0],
                                        _stream(stream))
    _ok(rc, "mep_dispatch_int8_smooth")
    return recv, recv_scale


def mep_dispatch_int8_smooth_workspace_size(T: int, K: int) -> int:
    """Bytes of scratch mep_dispatch_int8_smooth_grouped needs (the sorted slot list)."""
    return int(lib().mep_dispatch_int8_smooth_workspace_size(T, K))


def mep_dispatch_int8_smooth_grouped(x: torch.Tensor, ids: torch.Tensor, pos: torch.Tensor, K: int,
                                     smooth: torch.Tensor, recv: torch.Tensor, recv_scale: torch.Tensor,
                                     workspace: Optional[torch.Tensor] = None, stream=None):
    """mep_dispatch_int8_smooth with the slots taken in expert order within chunks of
    tokens (same codes and scales). ``workspace``: a uint8 device tensor of at least
    mep_dispatch_int8_smooth_workspace_size(T, K) bytes; allocated here when None."""
    T, H = x.shape
    _need(ids.numel() == T * K and pos.numel() == T * K, "ids and pos must hold T*K slots")
    _need(smooth.dim() == 2 and smooth.shape[1] == H, "smooth must be [experts, H]")
    _need(recv.dim() == 2 and recv.shape[1] == H and _n(recv_scale) >= recv.shape[0],
          "recv [rows, H] and recv_scale [rows] needed")
    need = mep_dispatch_int8_smooth_workspace_size(T, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _need(workspace.numel() * workspace.element_size() >= need, "workspace too small")
    rc = lib().mep_dispatch_int8_smooth_grouped(_ptr(x, torch.bfloat16, "x"), _ptr(ids, torch.int32, "ids"),
                                                _ptr(pos, torch.int32, "pos"), T, K, H,
                                                _ptr(smooth, torch.float32, "smooth"), smooth.shape[0],
                                                _ptr(recv, torch.int8, "recv"),
                                                _ptr(recv_scale, torch.float32, "recv_scale"), recv.shape[0],
                                                _ptr(workspace, None, "workspace"),
                                                workspace.numel() * workspace.element_size(), _stream(stream))
    _ok(rc, "mep_dispatch_int8_smooth_grouped")
    return recv, recv_scale


MEP_PLAN_STATIC_WS_BYTES = 4 << 20


def mep_plan_static_ws(ids: torch.Tensor, R: int, n_keys: int, S: int, K: int, out: PlanBuffers,
                       mode: int = MEP_PLAN_BALANCED, keys_per_rank: int = 0,
                       keep: Optional[torch.Tensor] = None, stream=None) -> PlanBuffers:
    """mep_plan for callers that cannot allocate device memory: the scratch is a 4 MiB
    array inside libmep (``out.workspace`` is not used). See include/mep.h."""
    f = lib().mep_plan_static_ws
    if ids.numel() != R * S * K:
        raise ValueError("ids must hold R*S*K slots")
    _need(keep is None or keep.numel() == R * S * K, "keep must hold R*S*K flags")
    _check_plan_buffers(out, R, n_keys, R * S * K)
    rc = f(_ptr(ids, torch.int32, "ids"), _ptr(keep, torch.uint8, "keep"), R, n_keys, S, K, mode,
           keys_per_rank, _ptr(out.pos), _ptr(out.hist), _ptr(out.rank_off), _ptr(out.load),
           _ptr(out.rep_count), _ptr(out.rep_key), _ptr(out.rep_cu), _ptr(out.stats),
           _stream(stream))
    _ok(rc, "mep_plan_static_ws")
    return out



@dataclasses.dataclass
class RouteBuffers:
    """Device buffers of one routing round trip from host memory (mep_route_host)."""

    R: int
    E: int
    S: int
    K: int
    H: int
    quant: int
    ids: torch.Tensor                   # int32 [N]
    gates: torch.Tensor                 # fp32 [N]
    x: torch.Tensor                     # bf16 [T, H]
    recv: torch.Tensor                  # bf16 or int8 [N, H]
    recv_scale: Optional[torch.Tensor]  # fp32 [N] (int8)
    out: torch.Tensor                   # bf16 [T, H]
    plan: PlanBuffers

    @staticmethod
    def allocate(R: int, E: int, S: int, K: int, H: int, quant: int = 0, device=None) -> "RouteBuffers":
        dev = device or torch.device("cuda", torch.cuda.current_device())
        T, N = R * S, R * S * K
        return RouteBuffers(
            R, E, S, K, H, quant,
            torch.empty(N, dtype=torch.int32, device=dev), torch.empty(N, dtype=torch.float32, device=dev),
            torch.empty((T, H), dtype=torch.bfloat16, device=dev),
            torch.empty((N, H), dtype=torch.int8 if quant else torch.bfloat16, device=dev),
            torch.empty(N, dtype=torch.float32, device=dev) if quant else None,
            torch.empty((T, H), dtype=torch.bfloat16, device=dev),
            PlanBuffers.allocate(R, E, S, K, dev))

    def c_struct(self) -> _RouteBuffersC:
        p = lambda t: None if t is None else t.data_ptr()
        pb = self.plan
        return _RouteBuffersC(self.R, self.E, self.S, self.K, self.H, self.quant, p(self.ids), p(self.gates),
                              p(self.x), p(self.recv), p(self.recv_scale), p(self.out), p(pb.pos), p(pb.hist),
                              p(pb.rank_off), p(pb.load), p(pb.rep_count), p(pb.rep_key), p(pb.rep_cu),
                              p(pb.stats), p(pb.workspace), pb.workspace.numel())


def _host_ptr(t: torch.Tensor, dtype, name: str):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def mep_route_host(rb: RouteBuffers, ids_h: torch.Tensor, gates_h: torch.Tensor, x_h: torch.Tensor,
                   out_h: torch.Tensor, stream=None, c_struct: Optional[_RouteBuffersC] = None) -> torch.Tensor:
    """Upload, plan, dispatch, combine (identity expert), download: one C call, all
    enqueued on `stream`. Pinned host tensors keep it asynchronous."""
    T, N = rb.R * rb.S, rb.R * rb.S * rb.K
    if ids_h.numel() != N or gates_h.numel() != N or tuple(x_h.shape) != (T, rb.H) or tuple(out_h.shape) != (T, rb.H):
        raise ValueError("host tensors must match the buffers' shapes")
    cs = c_struct if c_struct is not None else rb.c_struct()
    rc = lib().mep_route_host(ctypes.byref(cs), _host_ptr(ids_h, torch.int32, "ids_h"),
                              _host_ptr(gates_h, torch.float32, "gates_h"), _host_ptr(x_h, torch.bfloat16, "x_h"),
                              _host_ptr(out_h, torch.bfloat16, "out_h"), _stream(stream))
    _ok(rc, "mep_route_host")
    return out_h
