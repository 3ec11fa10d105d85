"""The C-ABI library on a machine without a GPU: it builds, loads, exports every
function include/mep.h declares, and rejects bad arguments with the documented status
before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mep.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mep_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from dispatch_combine_topk_b200 import build
    build.build()
    import dispatch_combine_topk_b200 as mep
    return mep.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"mep_plan", "mep_update_expert", "mep_dispatch", "mep_combine", "mep_histogram",
            "mep_plan_workspace_size", "mep_get_error", "mep_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    assert L.mep_version() >> 16 == 1
    for code in range(8):
        assert L.mep_status_string(code) and b"unknown" not in L.mep_status_string(code)
    assert b"unknown" in L.mep_status_string(99)


FAKE = ctypes.c_void_p(0x1000)   # never dereferenced: every call below fails its checks


def test_plan_argument_checks(L):
    P = FAKE
    args = lambda **kw: dict(dict(ids=P, keep=None, R=2, E=4, S=2, K=2, mode=0, kpr=0,
                                  ws=P, wsb=1 << 20), **kw)

    def call(a):
        return L.mep_plan(a["ids"], a["keep"], a["R"], a["E"], a["S"], a["K"], a["mode"], a["kpr"],
                          P, P, P, None, P, P, P, P, a["ws"], a["wsb"], None)
    assert call(args(ids=None)) == 1                      # NULLPTR
    assert call(args(R=0)) == 3                           # SHAPE
    assert call(args(K=33)) == 3
    assert call(args(E=5000)) == 3
    assert call(args(R=1 << 16, S=1 << 16)) == 3          # N >= 2^31
    assert call(args(E=5)) == 4                           # VALUE: E % R != 0
    assert call(args(keep=P)) == 4                        # VALUE: mask in balanced mode
    assert call(args(mode=7)) == 4
    assert call(args(mode=1, kpr=3)) == 4                 # kpr * R != n_keys
    assert call(args(ws=None)) == 5                       # WORKSPACE
    assert call(args(wsb=8)) == 5
    assert call(args(ws=ctypes.c_void_p(0x1008))) == 5    # not 256-byte aligned
    assert L.mep_plan_workspace_size(8, 64, 4096, 8) >= 128 * 64 * 4


def test_update_expert_argument_checks(L):
    P = FAKE

    def call(scales=None, thr=None, act=None, BS=4, K=2, E=8, F=2, rank=0, ws=2, mode=0):
        return L.mep_update_expert(P, P, scales, thr, act, BS, K, E, F, rank, ws, mode, P, P, None)
    assert call(scales=P) == 1
    assert call(thr=P) == 1
    assert call(act=P) == 1
    assert call(K=17) == 3
    assert call(E=1025) == 3
    assert call(K=3, E=2) == 3
    assert call(F=4) == 3            # F > world_size + 1
    assert call(mode=2) == 4
    assert call(ws=769) == 4
    assert call(rank=2) == 4
    assert call(ws=1) == 4           # F=2 <= ws+1 is fine; ws < 2 in mode 0 -> VALUE


def test_update_expert_ranks_argument_checks(L):
    P = FAKE

    def call(scales=None, thr=None, act=None, BS=4, K=2, E=8, F=2, ws=2, mode=0):
        return L.mep_update_expert_ranks(P, P, scales, thr, act, BS, K, E, F, ws, mode, P, P, None)
    assert call(scales=P) == 1
    assert call(act=P) == 1
    assert call(BS=0) == 3
    assert call(K=3, E=2) == 3
    assert call(F=4) == 3
    assert call(mode=2) == 4
    assert call(ws=1) == 4
    assert call(BS=1 << 25, K=16, ws=8) == 3      # rows * K past int32


def test_dedup_and_expand_argument_checks(L):
    P = FAKE
    wsb = L.mep_dedup_workspace_size(8, 4096, 8)
    assert wsb >= 8 * 4096 * 8 * 5
    assert L.mep_dedup_workspace_size(0, 1, 1) == 0

    def dedup(pos=P, R=2, S=4, K=2, ws=P, wsb=1 << 20, out=P):
        return L.mep_dedup_plan(pos, P, R, S, K, out, P, P, P, P, ws, wsb, None)
    assert dedup(pos=None) == 1
    assert dedup(out=None) == 1
    assert dedup(R=0) == 3
    assert dedup(K=33) == 3
    assert dedup(R=5000) == 3
    assert dedup(R=1 << 16, S=1 << 16) == 3
    assert dedup(ws=None) == 5
    assert dedup(wsb=16) == 5
    assert dedup(ws=ctypes.c_void_p(0x1008)) == 5

    def expand(src=P, ss=None, src_rows=4, gidx=P, rows=4, H=8, quant=0, dst=P, ds=None):
        return L.mep_expand(src, ss, src_rows, gidx, rows, H, quant, dst, ds, None)
    assert expand(quant=2) == 2
    assert expand(rows=-1) == 3
    assert expand(H=0) == 3
    assert expand(rows=0) == 0                  # nothing to do: no launch
    assert expand(gidx=None) == 1
    assert expand(quant=1, ss=P) == 1           # int8 rows need both scale arrays
    assert expand(quant=1, ds=P) == 1


def test_dispatch_combine_argument_checks(L):
    P = FAKE
    assert L.mep_dispatch(P, P, 4, 2, 64, 2, P, P, 8, None) == 2         # DTYPE
    assert L.mep_dispatch(None, P, 4, 2, 64, 0, P, None, 8, None) == 1   # NULLPTR
    assert L.mep_dispatch(P, P, 4, 2, 64, 1, P, None, 8, None) == 1      # int8 without scales
    assert L.mep_dispatch(P, P, 4, 0, 64, 0, P, None, 8, None) == 3
    assert L.mep_dispatch(P, P, 4, 2, 0, 0, P, None, 8, None) == 3
    assert L.mep_dispatch(P, P, 0, 2, 64, 0, P, None, 8, None) == 0      # empty: no launch
    assert L.mep_combine(P, 8, None, P, 4, 2, 64, P, None) == 1
    assert L.mep_combine(P, 8, P, P, 4, 33, 64, P, None) == 3
    assert L.mep_combine(P, -1, P, P, 4, 2, 64, P, None) == 3
    assert L.mep_combine(P, 8, P, P, 0, 2, 64, P, None) == 0
    assert L.mep_histogram(P, 10, 0, P, None) == 3
    assert L.mep_histogram(P, 10, 4, None, None) == 1
    assert L.mep_dequantize(None, P, 4, 8, P, None) == 1
    assert L.mep_get_error(None, None, 0) == 1
    L.mep_selftest_bounded_wait.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    assert L.mep_selftest_bounded_wait(10, None, None) == 1
    assert L.mep_selftest_bounded_wait(0, P, None) == 4
    assert L.mep_selftest_bounded_wait(1 << 23, P, None) == 4


def test_smooth_dispatch_grouped_argument_checks(L):
    P = FAKE
    c_size = ctypes.c_size_t
    L.mep_dispatch_int8_smooth_workspace_size.argtypes = [ctypes.c_int64, ctypes.c_int32]
    L.mep_dispatch_int8_smooth_workspace_size.restype = c_size
    assert L.mep_dispatch_int8_smooth_workspace_size(1000, 8) == 32000
    assert L.mep_dispatch_int8_smooth_workspace_size(3, 3) == 256          # 256-byte multiples
    assert L.mep_dispatch_int8_smooth_workspace_size(0, 8) == 0
    assert L.mep_dispatch_int8_smooth_workspace_size(-1, 8) == 0
    assert L.mep_dispatch_int8_smooth_workspace_size(4, 0) == 0
    i64, i32 = ctypes.c_int64, ctypes.c_int32
    L.mep_dispatch_int8_smooth_grouped.argtypes = [ctypes.c_void_p] * 3 + [i64, i32, i64, ctypes.c_void_p, i32,
                                                   ctypes.c_void_p, ctypes.c_void_p, i64, ctypes.c_void_p, c_size,
                                                   ctypes.c_void_p]
    W = ctypes.c_void_p(0x100000)                                          # 256-byte aligned, never read

    def call(x=P, T=4, K=2, H=64, E=3, rows=8, ws=W, nbytes=256):
        return L.mep_dispatch_int8_smooth_grouped(x, P, P, T, K, H, P, E, P, P, rows, ws, nbytes, None)
    assert call(x=None) == 1                                               # NULLPTR
    assert call(K=0) == 3 and call(K=33) == 3 and call(H=0) == 3 and call(E=0) == 3 and call(rows=-1) == 3
    assert call(ws=None) == 5                                              # WORKSPACE: missing
    assert call(nbytes=16) == 5                                            # too small
    assert call(ws=ctypes.c_void_p(0x100010)) == 5                         # not 256-byte aligned
    assert call(T=0, ws=None, nbytes=0) == 0                               # empty: no launch, no workspace


def test_route_buffers_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes mirror of mep_route_buffers_t has the header's layout
    (size and field offsets as gcc lays the struct out)."""
    import subprocess
    import dispatch_combine_topk_b200 as mep
    C = mep._RouteBuffersC
    names = [f[0] for f in C._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"mep.h\"\nint main(void){\n"
                   "printf(\"%zu\\n\", sizeof(mep_route_buffers_t));\n" +
                   "".join(f'printf("%zu\\n", offsetof(mep_route_buffers_t, {n}));\n' for n in names) +
                   "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(C)
    assert got[1:] == [getattr(C, n).offset for n in names]


def test_route_host_argument_checks(L):
    import dispatch_combine_topk_b200 as mep
    P = FAKE
    b = mep._RouteBuffersC(2, 4, 2, 2, 8, 0, *([0x1000] * 15), 1 << 20)
    assert L.mep_route_host(None, P, P, P, P, None) == 1
    assert L.mep_route_host(ctypes.byref(b), None, P, P, P, None) == 1
    b.quant = 3
    assert L.mep_route_host(ctypes.byref(b), P, P, P, P, None) == 2
    b.quant, b.R = 0, 0
    assert L.mep_route_host(ctypes.byref(b), P, P, P, P, None) == 3
    b.R, b.ids = 2, None
    assert L.mep_route_host(ctypes.byref(b), P, P, P, P, None) == 1


def test_stream_synchronize_timeout_argument_check(L):
    assert L.mep_stream_synchronize_timeout(None, -1) == 4


def test_maxvio_from_a_plan_summary(L, golden_dir):
    """mep_maxvio is host arithmetic: on the plan hand example it gives the golden's
    maxvio before (0.5) and after (0.0); on every balanced workload's oracle plan the
    after-value is 0; an empty plan has no expert-level value; bad sizes are refused."""
    import json
    import math
    import dispatch_combine_topk_b200 as mep
    import oracle
    import synth
    g = json.load(open(os.path.join(golden_dir, "plan_hand_r2_e4_s2_k2.json")))
    R, E, S, K = g["R"], g["E"], g["S"], g["K"]
    p = oracle.plan_balanced(__import__("numpy").array(g["ids"], "int32").ravel(), R, E, S, K)
    st = [p.max_load, p.max_chunk, p.redundant, p.prefetched, p.n_kept, p.max_hist, 0, 0]
    m = mep.mep_maxvio(st, S, K, E)
    assert m["rank_before"] == g["expected"]["maxvio_before"]
    assert m["rank_after"] == g["expected"]["maxvio_after"]
    assert m["expert"] == max(g["expected"]["hist"]) / (R * S * K / E) - 1.0
    for name in ("tiny", "r8"):
        w = synth.get(name)
        ids, _ = synth.router(w)
        p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
        st = [p.max_load, p.max_chunk, p.redundant, p.prefetched, p.n_kept, p.max_hist, 0, 0]
        m = mep.mep_maxvio(st, w.S, w.K, w.E)
        assert m["rank_after"] == 0.0 and m["rank_before"] == p.maxvio_before(w.S, w.K)
    assert math.isnan(mep.mep_maxvio([0] * 8, 2, 2, 4)["expert"])
    assert L.mep_maxvio(None, 2, 2, 4, None, None, None) == 1
    buf = (ctypes.c_int32 * 8)()
    assert L.mep_maxvio(ctypes.cast(buf, ctypes.c_void_p), 0, 2, 4, None, None, None) == 3


def test_static_ws_checks_arguments_before_its_size(L):
    """mep_plan_static_ws reports mep_plan's argument errors first: a call that is both
    invalid and larger than the 4 MiB array gets the argument's status, not
    MEP_ERR_WORKSPACE (which is only for a valid plan that does not fit)."""
    P = FAKE
    big = dict(R=8, E=2048, S=32768, K=8)          # 2^21 slots x 2048 keys: 8 MiB of scratch
    import dispatch_combine_topk_b200 as mep
    assert mep.mep_plan_workspace_size(big["R"], big["E"], big["S"], big["K"]) > 4 << 20

    def call(ids=P, keep=None, R=big["R"], E=big["E"], S=big["S"], K=big["K"], mode=0, kpr=0):
        return L.mep_plan_static_ws(ids, keep, R, E, S, K, mode, kpr, P, P, P, None, P, P, P, P, None)
    assert call(K=33) == 3                         # SHAPE, not WORKSPACE
    assert call(E=2047) == 4                       # VALUE: E % R != 0
    assert call(mode=9) == 4
    assert call(keep=P) == 4
    assert call(ids=None) == 1
    assert call() == 5                             # valid, too large: WORKSPACE


def test_plan_rank_argument_checks(L):
    P = FAKE

    def call(ids=P, hist=P, R=4, E=16, S=8, K=2, rank=0, ws=P, wsb=1 << 20):
        return L.mep_plan_rank(ids, hist, R, E, S, K, rank, P, P, P, P, P, ws, wsb, None)
    assert call(ids=None) == 1
    assert call(hist=None) == 1
    assert call(R=0) == 3
    assert call(K=33) == 3
    assert call(E=5000) == 3
    assert call(E=18) == 4                         # E % R != 0
    assert call(rank=4) == 4
    assert call(rank=-1) == 4
    assert call(ws=None) == 5
    assert call(wsb=16) == 5
    assert L.mep_plan_rank_workspace_size(0, 16, 8, 2) == 0
    assert L.mep_plan_rank_workspace_size(4, 16, 8, 2) > 0


def test_plan_launch_count(L):
    """Host-only query: one launch when the whole plan fits one launch (at most 16384
    slots and few enough keys for shared memory), three for the tiled sort."""
    L.mep_plan_launches.argtypes = [ctypes.c_int32] * 4
    L.mep_plan_launches.restype = ctypes.c_int32
    assert L.mep_plan_launches(4, 16, 128, 2) == 1            # tiny
    assert L.mep_plan_launches(8, 272, 256, 8) == 1           # mapping workload: 16384 slots
    assert L.mep_plan_launches(1, 2, 16385, 1) == 3           # one slot past the limit
    assert L.mep_plan_launches(64, 1536, 8, 8) == 3           # too many keys for one launch
    assert L.mep_plan_launches(32, 256, 8192, 8) == 3         # int8 workload
    assert L.mep_plan_launches(0, 16, 128, 2) == 0


def test_rank_buffer_calls_argument_checks(L):
    P = FAKE
    A = ctypes.c_void_p(0x2000)                        # 8-byte aligned stand-ins, never read
    assert L.mep_dispatch_ranks(P, P, 4, 2, 64, 2, A, None, 2, 8, None) == 2       # DTYPE
    assert L.mep_dispatch_ranks(None, P, 4, 2, 64, 0, A, None, 2, 8, None) == 1    # NULLPTR
    assert L.mep_dispatch_ranks(P, P, 4, 2, 64, 1, A, None, 2, 8, None) == 1       # int8 without scales
    assert L.mep_dispatch_ranks(P, P, 4, 2, 60, 0, A, None, 2, 8, None) == 3       # H % 8
    assert L.mep_dispatch_ranks(P, P, 4, 2, 64, 0, A, None, 0, 8, None) == 3       # R
    assert L.mep_dispatch_ranks(P, P, 4, 2, 64, 0, A, None, 2, 0, None) == 3       # rows per rank
    assert L.mep_dispatch_ranks(ctypes.c_void_p(0x1008), P, 4, 2, 64, 0, A, None, 2, 8, None) == 4  # x misaligned
    assert L.mep_dispatch_ranks(P, P, 0, 2, 64, 0, A, None, 2, 8, None) == 0       # empty: no launch
    assert L.mep_combine_ranks(A, None, 0, 2, 8, None, P, 4, 2, 64, P, None) == 1
    assert L.mep_combine_ranks(A, None, 1, 2, 8, P, P, 4, 2, 64, P, None) == 1     # int8 without scales
    assert L.mep_combine_ranks(A, A, 1, 2, 8, P, P, 4, 2, 72, P, None) == 3        # int8: H % 16
    assert L.mep_combine_ranks(A, None, 0, 2, 8, P, P, 4, 2, 64, ctypes.c_void_p(0x1004), None) == 4
    assert L.mep_combine_ranks(A, None, 0, 2, 8, P, P, 0, 2, 64, P, None) == 0
