"""Oracle for MoE expert-parallel token routing — TEST INFRASTRUCTURE ONLY.

A thin numpy front end over the plain C oracle in ``mep_oracle.c``. Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it;
the product path (the CUDA library and its Python binding) never does.

bf16 arrays are passed as their bit patterns in ``np.uint16`` arrays.
"""
from __future__ import annotations

import ctypes
import dataclasses

import numpy as np

from . import build as _build

_lib = None


def _configure(L):
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    L.orc_float_to_bf16.argtypes = [ctypes.c_float]
    L.orc_float_to_bf16.restype = ctypes.c_uint16
    L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_float.restype = ctypes.c_float
    L.orc_histogram.argtypes = [P, i64, i32, P]
    L.orc_plan_balanced.argtypes = [P, i32, i32, i32, i32, P, P, P, i32, P, P, P, P]
    L.orc_plan_grouped.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, P, i32, P, P, P, P]
    L.orc_update_expert.argtypes = [P, i64, i32, P, i32, i32, P, P, P, i64, i64, i64, P, P]
    L.orc_dispatch.argtypes = [P, P, i64, i32, i64, i64, P]
    L.orc_quantize_row.argtypes = [P, i64, P, P]
    L.orc_quantize_row.restype = None
    L.orc_dispatch_int8.argtypes = [P, P, i64, i32, i64, i64, P, P]
    L.orc_dequantize.argtypes = [P, P, i64, i64, P]
    L.orc_dequantize.restype = None
    L.orc_combine.argtypes = [P, i64, P, P, i64, i32, i64, P]
    L.orc_double_to_bf16.argtypes = [ctypes.c_double]
    L.orc_double_to_bf16.restype = ctypes.c_uint16
    L.orc_combine_add_rmsnorm.argtypes = [P, i64, P, P, i64, i32, i64, P, P, ctypes.c_double,
                                          P, P, P, P]
    L.orc_combine_add_rmsnorm.restype = ctypes.c_int
    L.orc_prefetch_plan.argtypes = [P, P, i32, i32, i32, i32, P, P]
    L.orc_dedup_plan.argtypes = [P, i64, i32, P, i32, P, P, P, P, P, i64]
    L.orc_expand.argtypes = [P, P, i64, P, i64, i64, P, P]
    L.orc_prefetch_weights.argtypes = [P, P, i32, i32, i32, i64, P]
    L.orc_grad_reduce.argtypes = [P, P, P, i32, i32, i32, i64]
    for name in ["orc_prefetch_plan", "orc_prefetch_weights", "orc_grad_reduce"]:
        getattr(L, name).restype = ctypes.c_int
    L.orc_dispatch_int8_smooth.argtypes = [P, P, P, i64, i32, i64, P, i32, i64, P, P]
    L.orc_dispatch_int8_smooth.restype = ctypes.c_int
    for name in ["orc_histogram", "orc_plan_balanced", "orc_plan_grouped",
                 "orc_update_expert", "orc_dispatch", "orc_dispatch_int8", "orc_combine"]:
        getattr(L, name).restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


class OracleError(RuntimeError):
    pass


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle returned {rc} ({'invalid argument' if rc == -1 else 'invalid data'})")


# ------------------------------------------------------------------------ bf16

def float_to_bf16(values) -> np.ndarray:
    """binary32 -> bf16 bits, round to nearest even (element by element)."""
    v = np.asarray(values, np.float32).ravel()
    L = lib()
    return np.array([L.orc_float_to_bf16(float(x)) for x in v], np.uint16).reshape(np.shape(values))


def bf16_to_float(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------- a1 / a2

def histogram(ids, E: int) -> np.ndarray:
    ids = _c(ids, np.int32).ravel()
    hist = np.zeros(E, np.int32)
    _check(lib().orc_histogram(_p(ids), ids.size, E, _p(hist)), "histogram")
    return hist


@dataclasses.dataclass
class Plan:
    pos: np.ndarray          # int32 [N], row of every slot (-1 = dropped)
    hist: np.ndarray         # int32 [n_keys]
    rank_off: np.ndarray     # int32 [R+1]
    rep_count: np.ndarray    # int32 [R]
    rep_key: np.ndarray      # int32 [R, cap], -1 past rep_count
    rep_cu: np.ndarray       # int32 [R, cap+1], zero past rep_count
    load: np.ndarray         # int32 [R]: rows per rank if nothing moved off its home
    max_load: int
    max_chunk: int
    redundant: int
    prefetched: int
    n_kept: int
    max_hist: int

    def maxvio_before(self, S: int, K: int) -> float:
        """max_load / mean_load - 1 with mean_load = S*K."""
        return self.max_load / float(S * K) - 1.0

    def maxvio_after(self, S: int, K: int) -> float:
        return self.max_chunk / float(S * K) - 1.0


def plan_balanced(ids, R: int, E: int, S: int, K: int) -> Plan:
    ids = _c(ids, np.int32).ravel()
    assert ids.size == R * S * K
    cap = E
    pos = np.empty(ids.size, np.int32)
    hist = np.empty(E, np.int32)
    load = np.empty(R, np.int32)
    rep_count = np.empty(R, np.int32)
    rep_key = np.empty((R, cap), np.int32)
    rep_cu = np.empty((R, cap + 1), np.int32)
    stats = np.zeros(8, np.int64)
    rc = lib().orc_plan_balanced(_p(ids), R, E, S, K, _p(pos), _p(hist), _p(load), cap,
                                 _p(rep_count), _p(rep_key), _p(rep_cu), _p(stats))
    _check(rc, "plan_balanced")
    rank_off = (np.arange(R + 1, dtype=np.int64) * S * K).astype(np.int32)
    return Plan(pos, hist, rank_off, rep_count, rep_key, rep_cu, load, *[int(s) for s in stats[:6]])


def plan_grouped(keys, keep, R: int, n_keys: int, keys_per_rank: int, S: int, K: int) -> Plan:
    keys = _c(keys, np.int32).ravel()
    keep = None if keep is None else _c(keep, np.uint8).ravel()
    cap = n_keys
    pos = np.empty(keys.size, np.int32)
    hist = np.empty(n_keys, np.int32)
    rank_off = np.empty(R + 1, np.int32)
    rep_count = np.empty(R, np.int32)
    rep_key = np.empty((R, cap), np.int32)
    rep_cu = np.empty((R, cap + 1), np.int32)
    stats = np.zeros(8, np.int64)
    rc = lib().orc_plan_grouped(_p(keys), _p(keep), R, n_keys, keys_per_rank, S, K, _p(pos),
                                _p(hist), _p(rank_off), cap, _p(rep_count), _p(rep_key),
                                _p(rep_cu), _p(stats))
    _check(rc, "plan_grouped")
    load = np.diff(rank_off).astype(np.int32)
    return Plan(pos, hist, rank_off, rep_count, rep_key, rep_cu, load, *[int(s) for s in stats[:6]])


# ------------------------------------------------------------------------- a3

def update_expert(expert_ids, eplb_table, expert_scales, pruning_threshold, active_mask,
                  local_rank_id: int, world_size: int, balance_mode: int):
    ids = _c(expert_ids, np.int32)
    BS, K = ids.shape
    table = _c(eplb_table, np.int32)
    E, F = table.shape
    sc = None if expert_scales is None else _c(expert_scales, np.float32)
    thr = None if pruning_threshold is None else _c(pruning_threshold, np.float32).ravel()
    act = None if active_mask is None else _c(active_mask, np.uint8).ravel()
    out_ids = np.empty((BS, K), np.int32)
    out_mask = np.empty((BS, K), np.uint8)
    rc = lib().orc_update_expert(_p(ids), BS, K, _p(table), E, F, _p(sc), _p(thr), _p(act),
                                 local_rank_id, world_size, balance_mode, _p(out_ids),
                                 _p(out_mask))
    _check(rc, "update_expert")
    return out_ids, out_mask.astype(bool)


# --------------------------------------------------------------------- a4 / a5

def dispatch(x_bits, pos, K: int, rows: int) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    pos = _c(pos, np.int32).ravel()
    recv = np.zeros((rows, H), np.uint16)
    _check(lib().orc_dispatch(_p(x), _p(pos), T, K, H, rows, _p(recv)), "dispatch")
    return recv


def quantize_row(x_bits):
    x = _c(x_bits, np.uint16).ravel()
    q = np.empty(x.size, np.int8)
    s = np.zeros(1, np.float32)
    lib().orc_quantize_row(_p(x), x.size, _p(q), _p(s))
    return q, s[0]


def dispatch_int8(x_bits, pos, K: int, rows: int):
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    pos = _c(pos, np.int32).ravel()
    q = np.zeros((rows, H), np.int8)
    sc = np.zeros(rows, np.float32)
    _check(lib().orc_dispatch_int8(_p(x), _p(pos), T, K, H, rows, _p(q), _p(sc)), "dispatch_int8")
    return q, sc


def dequantize(q, scale) -> np.ndarray:
    q = _c(q, np.int8)
    rows, H = q.shape
    scale = _c(scale, np.float32).ravel()
    y = np.empty((rows, H), np.uint16)
    lib().orc_dequantize(_p(q), _p(scale), rows, H, _p(y))
    return y


def combine(y_bits, pos, gates, K: int) -> np.ndarray:
    y = _c(y_bits, np.uint16)
    rows, H = y.shape
    pos = _c(pos, np.int32).ravel()
    gates = _c(gates, np.float32).ravel()
    T = pos.size // K
    out = np.empty((T, H), np.uint16)
    _check(lib().orc_combine(_p(y), rows, _p(pos), _p(gates), T, K, H, _p(out)), "combine")
    return out


def combine_int8(q, scale, pos, gates, K: int) -> np.ndarray:
    """Combine of int8 rows with per-row scales: by definition the combine of the
    dequantised rows, y = bf16(fl(q * scale)) (the two oracle steps, composed)."""
    return combine(dequantize(q, scale), pos, gates, K)


def route_tokens(x_bits, kept, gates, K: int, quant: int = 0) -> np.ndarray:
    """Dispatch -> identity expert -> combine for a few tokens, one token at a time.

    ``kept`` is a bool [n, K] array (slot kept or dropped). Each token is run as its
    own small problem through the oracle's own dispatch, dequantisation and combine,
    with its kept slots on rows 0..K-1; used to check single tokens of a workload too
    large to route whole on the host.
    """
    x = _c(x_bits, np.uint16)
    n, H = x.shape
    out = np.empty((n, H), np.uint16)
    for i in range(n):
        pos = np.where(np.asarray(kept[i], bool), np.arange(K, dtype=np.int32), -1).astype(np.int32)
        if quant:
            q, sc = dispatch_int8(x[i:i + 1], pos, K, K)
            y = dequantize(q, sc)
        else:
            y = dispatch(x[i:i + 1], pos, K, K)
        out[i] = combine(y, pos, np.asarray(gates[i], np.float32), K)[0]
    return out


def double_to_bf16(values) -> np.ndarray:
    """binary64 -> bf16 bits, round to nearest even, in one rounding (element by element)."""
    v = np.asarray(values, np.float64).ravel()
    L = lib()
    return np.array([L.orc_double_to_bf16(float(x)) for x in v], np.uint16).reshape(np.shape(values))


def combine_add_rmsnorm(y_bits, pos, gates, K: int, residual_bits, gamma_bits, eps: float):
    """Combine, residual add and RMSNorm. Returns (x_out bits, y_out bits, y_exact
    float64 [T,H], rstd float64 [T])."""
    y = _c(y_bits, np.uint16)
    rows, H = y.shape
    pos = _c(pos, np.int32).ravel()
    gates = _c(gates, np.float32).ravel()
    T = pos.size // K
    res = _c(residual_bits, np.uint16)
    gam = _c(gamma_bits, np.uint16).ravel()
    x_out = np.empty((T, H), np.uint16)
    y_out = np.empty((T, H), np.uint16)
    y_exact = np.empty((T, H), np.float64)
    rstd = np.empty(T, np.float64)
    rc = lib().orc_combine_add_rmsnorm(_p(y), rows, _p(pos), _p(gates), T, K, H, _p(res), _p(gam),
                                       float(eps), _p(x_out), _p(y_out), _p(y_exact), _p(rstd))
    _check(rc, "combine_add_rmsnorm")
    return x_out, y_out, y_exact, rstd


# --------------------------------------------------------------------- f2 / f3

def prefetch_plan(rep_count, rep_key, R: int, E: int, B: int):
    """Slot of every prefetched replica and the weight row every replica reads.
    Returns (slot_expert int32 [R, B], rep_weight int32 [R, cap])."""
    rep_count = _c(rep_count, np.int32).ravel()
    rep_key = _c(rep_key, np.int32)
    cap = rep_key.shape[1]
    slot_expert = np.empty((R, B), np.int32)
    rep_weight = np.empty((R, cap), np.int32)
    _check(lib().orc_prefetch_plan(_p(rep_count), _p(rep_key), R, E, cap, B, _p(slot_expert),
                                   _p(rep_weight)), "prefetch_plan")
    return slot_expert, rep_weight


def prefetch_weights(w_home_bits, slot_expert, R: int, B: int, w_slots_bits=None):
    w_home = _c(w_home_bits, np.uint16)
    E = w_home.shape[0]
    D = int(np.prod(w_home.shape[1:]))
    se = _c(slot_expert, np.int32).ravel()
    out = (np.zeros((R * B,) + w_home.shape[1:], np.uint16) if w_slots_bits is None
           else np.array(w_slots_bits, np.uint16, copy=True))
    _check(lib().orc_prefetch_weights(_p(w_home), _p(se), E, R, B, D, _p(out)), "prefetch_weights")
    return out


def grad_reduce(grad_home, grad_slots, slot_expert, R: int, B: int):
    """Returns (new grad_home, new grad_slots) as float32 copies."""
    gh = np.array(grad_home, np.float32, copy=True, order="C")
    gs = np.array(grad_slots, np.float32, copy=True, order="C")
    E = gh.shape[0]
    D = int(np.prod(gh.shape[1:]))
    se = _c(slot_expert, np.int32).ravel()
    _check(lib().orc_grad_reduce(_p(gh), _p(gs), _p(se), E, R, B, D), "grad_reduce")
    return gh, gs


def dispatch_int8_smooth(x_bits, ids, pos, K: int, smooth, rows: int):
    """int8 dispatch with per-expert smoothing scales: codes and scale per slot."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    ids = _c(ids, np.int32).ravel()
    pos = _c(pos, np.int32).ravel()
    sm = _c(smooth, np.float32)
    q = np.zeros((rows, H), np.int8)
    sc = np.zeros(rows, np.float32)
    _check(lib().orc_dispatch_int8_smooth(_p(x), _p(ids), _p(pos), T, K, H, _p(sm), sm.shape[0], rows,
                                          _p(q), _p(sc)), "dispatch_int8_smooth")
    return q, sc


@dataclasses.dataclass
class Dedup:
    """One row per (token, destination rank): the send list, every slot's row, the
    ranks' first rows, the token of every row and every plan row's source row."""
    dsend: np.ndarray      # int32 [N]
    dpos: np.ndarray       # int32 [N]
    drank_off: np.ndarray  # int32 [R+1]
    dtok: np.ndarray       # int32 [N] (-1 past drank_off[R])
    gidx: np.ndarray       # int32 [len(pos)] (-1 past rank_off[R])


def dedup_plan(pos, K: int, rank_off) -> Dedup:
    pos = _c(pos, np.int32).ravel()
    rank_off = _c(rank_off, np.int32).ravel()
    N = pos.size
    R = rank_off.size - 1
    out = Dedup(np.empty(N, np.int32), np.empty(N, np.int32), np.empty(R + 1, np.int32),
                np.empty(N, np.int32), np.empty(N, np.int32))
    _check(lib().orc_dedup_plan(_p(pos), N, K, _p(rank_off), R, _p(out.dsend), _p(out.dpos),
                                _p(out.drank_off), _p(out.dtok), _p(out.gidx), N), "dedup_plan")
    return out


def expand(src, gidx, rows: int, src_scale=None, dst=None, dst_scale=None):
    """dst[p] = src[gidx[p]] for gidx[p] >= 0 (rows of any dtype; scales optional).
    Returns dst (and dst_scale when scales are given)."""
    src = np.ascontiguousarray(src)
    gidx = _c(gidx, np.int32).ravel()
    out = np.zeros((rows,) + src.shape[1:], src.dtype) if dst is None else np.array(dst, copy=True)
    row_bytes = int(src.dtype.itemsize * np.prod(src.shape[1:]))
    sc_in = None if src_scale is None else _c(src_scale, np.float32)
    sc_out = None
    if sc_in is not None:
        sc_out = np.zeros(rows, np.float32) if dst_scale is None else np.array(dst_scale, np.float32, copy=True)
    _check(lib().orc_expand(_p(src), None if sc_in is None else _p(sc_in), src.shape[0], _p(gidx), rows,
                            row_bytes, _p(out), None if sc_out is None else _p(sc_out)), "expand")
    return out if sc_out is None else (out, sc_out)
