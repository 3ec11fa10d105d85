"""GPU parity of dispatch (bf16 and int8), dequantisation and combine against the
oracle, element by element: at small sizes (several CTAs, ragged rows), and at the full
workload sizes, where the receive buffer is compared one rank partition at a time and
the combine output one chunk of tokens at a time, to bound host memory. Properties that
hold at any size (checksums of every row, closed forms) are checked as well."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced, gpu_plan_grouped

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("T,K,H", [(1, 1, 8), (37, 3, 256), (64, 8, 4096), (5, 32, 72),
                                   (33, 2, 7), (12, 4, 130), (300, 6, 7168)])
@pytest.mark.parametrize("quant", [0, 1])
def test_dispatch_combine_small_exact(T, K, H, quant):
    rng = np.random.default_rng(T * 100 + K * 10 + H + quant)
    rows = T * K + 3
    pos = rng.permutation(rows)[: T * K].astype(np.int32)
    pos[rng.random(T * K) < 0.15] = -1
    x = _rand_bf16((T, H), T + H, scale=float(rng.uniform(0.01, 50)))
    gates = rng.random(T * K).astype(np.float32)
    xb = bits(x)
    x_d, pos_d = x.to(dev()), torch.from_numpy(pos).to(dev())
    if quant == 0:
        recv = torch.zeros((rows, H), dtype=torch.bfloat16, device=dev())
        mep.mep_dispatch(x_d, pos_d, K, recv)
        ref = oracle.dispatch(xb, pos, K, rows)
        assert np.array_equal(bits(recv), ref)
        y_d, y_ref = recv, ref
    else:
        recv = torch.zeros((rows, H), dtype=torch.int8, device=dev())
        sc = torch.zeros(rows, dtype=torch.float32, device=dev())
        mep.mep_dispatch(x_d, pos_d, K, recv, sc, quant=1)
        q_ref, s_ref = oracle.dispatch_int8(xb, pos, K, rows)
        assert np.array_equal(recv.cpu().numpy(), q_ref)
        assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        y_d = torch.empty((rows, H), dtype=torch.bfloat16, device=dev())
        mep.mep_dequantize(recv, sc, y_d)
        y_ref = oracle.dequantize(q_ref, s_ref)
        assert np.array_equal(bits(y_d), y_ref)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(y_d, pos_d, torch.from_numpy(gates).to(dev()), K, out)
    assert np.array_equal(bits(out), oracle.combine(y_ref, pos, gates, K))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5, 6, 8, 16, 32])
def test_combine_random_rows_every_k(K):
    """Arbitrary expert rows (not copies of the token) and every K: catches a slot that
    reads the wrong row or sums in another order."""
    rng = np.random.default_rng(K)
    T, H, rows = 97, 1024, 500
    y = _rand_bf16((rows, H), 100 + K)
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.1] = -1
    gates = (rng.standard_normal(T * K) * 3).astype(np.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(y.to(dev()), torch.from_numpy(pos).to(dev()), torch.from_numpy(gates).to(dev()), K, out)
    assert np.array_equal(bits(out), oracle.combine(bits(y), pos, gates, K))


def test_quant_edge_rows():
    """Zero rows (scale 0), exact ties (scale 1), outliers, denormal-range values: rows
    whose scale is subnormal with 1/scale finite or overflowing, and the largest bf16."""
    H, K = 64, 2
    T = 8
    x = torch.zeros((T, H), dtype=torch.float32)
    x[1, :12] = torch.tensor([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 0.0, 126.5, -127.0, 0.25])
    x[2] = torch.linspace(-3000, 3000, H)
    x[3] = torch.linspace(-1e-37, 1e-37, H)
    x[4] = torch.linspace(-1e-36, 1e-36, H)          # scale subnormal, 1/scale finite
    x[5] = torch.linspace(-4e-37, 4e-37, H)          # scale close to where 1/scale overflows
    x[6, :3] = torch.tensor([9.2e-41, -1.84e-40, 0.0])  # bf16 subnormals: 1/scale overflows
    x[7] = torch.linspace(-1.0, 1.0, H) * 3.38e38    # near the largest finite bf16
    xb16 = x.to(torch.bfloat16)
    pos = np.arange(T * K, dtype=np.int32)
    recv = torch.zeros((T * K, H), dtype=torch.int8, device=dev())
    sc = torch.zeros(T * K, dtype=torch.float32, device=dev())
    mep.mep_dispatch(xb16.to(dev()), torch.from_numpy(pos).to(dev()), K, recv, sc, quant=1)
    q_ref, s_ref = oracle.dispatch_int8(bits(xb16), pos, K, T * K)
    assert np.array_equal(recv.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert recv[0:2].abs().max().item() == 0 and sc[0].item() == 0.0   # token 0: zero row


def test_row_out_of_range_is_skipped_and_flagged():
    T, K, H = 4, 2, 64
    x = _rand_bf16((T, H), 1).to(dev())
    pos = torch.tensor([0, 1, 2, 3, 4, 5, 6, 99], dtype=torch.int32, device=dev())
    recv = torch.zeros((T * K + 4, H), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x, pos, K, recv[: T * K])
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE
    assert recv[T * K:].abs().max().item() == 0   # guard rows untouched
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(recv[: T * K], pos, torch.ones(T * K, device=dev()), K, out)
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE


def test_empty_inputs():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    pos = torch.empty(0, dtype=torch.int32, device=dev())
    recv = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x, pos, 4, recv)
    out = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(recv, pos, torch.empty(0, device=dev()), 4, out)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- full workloads

def _route_full(name):
    """Plan + dispatch (+ dequant) + combine of a whole workload on the GPU, exactly as
    bench.py launches it."""
    w = synth.get(name)
    ids, gates = synth.router(w)
    x = synth.hidden(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    x_d = x.to(dev())
    g_d = torch.from_numpy(gates).to(dev())
    if w.quant:
        recv = torch.empty((w.N, w.H), dtype=torch.int8, device=dev())
        sc = torch.empty(w.N, dtype=torch.float32, device=dev())
        mep.mep_dispatch(x_d, pb.pos, w.K, recv, sc, quant=1)
        y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev())
        mep.mep_dequantize(recv, sc, y)
    else:
        recv, sc = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev()), None
        mep.mep_dispatch(x_d, pb.pos, w.K, recv)
        y = recv
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(y, pb.pos, g_d, w.K, out)
    torch.cuda.synchronize()
    return w, ids, gates, x, x_d, pb, recv, sc, y, out


def _row_checksum(t, chunk=32768):
    """Per-row sum of the raw 16-bit (or 8-bit) patterns, on the device, in row chunks
    (int32 is exact: |sum| <= 32768 * H)."""
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    out = torch.empty(t.shape[0], dtype=torch.int32, device=t.device)
    for i in range(0, t.shape[0], chunk):
        out[i:i + chunk] = t[i:i + chunk].to(torch.int32).sum(1, dtype=torch.int32)
    return out


# The oracle's calls release the GIL (ctypes), so independent partitions and chunks run
# on several host threads; each call is still the oracle's own single-threaded code.
_POOL = 8


def _oracle_partition(xb, pos, K, quant, lo, hi):
    """The oracle's dispatch restricted to the receive rows [lo, hi) (one rank's
    partition): the tokens with a slot there, their slots' rows shifted by lo, every
    other slot dropped."""
    inside = (pos >= lo) & (pos < hi)
    toks = np.unique(np.flatnonzero(inside) // K)
    pos_r = np.where(inside, pos - lo, -1).astype(np.int32).reshape(-1, K)[toks]
    if quant:
        return oracle.dispatch_int8(xb[toks], pos_r, K, hi - lo)
    return oracle.dispatch(xb[toks], pos_r, K, hi - lo)


def _assert_partitions_equal(xb, pos, K, quant, recv, sc, R, SK):
    def one(r):
        lo, hi = r * SK, (r + 1) * SK
        ref = _oracle_partition(xb, pos, K, quant, lo, hi)
        if quant:
            q_ref, s_ref = ref
            assert np.array_equal(recv[lo:hi].cpu().numpy(), q_ref), f"codes of rank {r}"
            assert np.array_equal(sc[lo:hi].cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), \
                f"scales of rank {r}"
        else:
            assert np.array_equal(bits(recv[lo:hi]), ref), f"rows of rank {r}"
        return r
    with ThreadPoolExecutor(_POOL) as ex:
        assert sorted(ex.map(one, range(R))) == list(range(R))


def _oracle_route_chunk(xb, gates, K, quant, t0, t1):
    """The oracle's dispatch -> identity expert -> combine for tokens [t0, t1), every
    slot kept, the chunk's slots on their own rows (the rows' order does not change any
    token's sum)."""
    n = t1 - t0
    pos_l = np.arange(n * K, dtype=np.int32)
    g = gates[t0:t1]
    if quant:
        q, s = oracle.dispatch_int8(xb[t0:t1], pos_l, K, n * K)
        return oracle.combine_int8(q, s, pos_l, g, K)
    return oracle.combine(oracle.dispatch(xb[t0:t1], pos_l, K, n * K), pos_l, g, K)


def _assert_combine_equal(xb, gates, K, quant, out, T, chunk=4096):
    def one(t0):
        t1 = min(T, t0 + chunk)
        ref = _oracle_route_chunk(xb, gates, K, quant, t0, t1)
        assert np.array_equal(bits(out[t0:t1]), ref), f"combine, tokens [{t0}, {t1})"
        return t1 - t0
    with ThreadPoolExecutor(_POOL) as ex:
        assert sum(ex.map(one, range(0, T, chunk))) == T


@pytest.mark.parametrize("name", ["r8", "skew", "int8"])
def test_full_workload_every_element(name):
    """The whole workload as bench.py launches it: every plan row, every element of the
    receive buffer (codes and scale bits for int8), every combine output, against the
    oracle. For int8 the combine here is mep_combine on mep_dequantize's rows; the fused
    combine of the int8 rows has its own test below."""
    w, ids, gates, x, x_d, pb, recv, sc, y, out = _route_full(name)
    assert mep.mep_get_error() == 0
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    pos = pb.pos.cpu().numpy()
    assert np.array_equal(pos, p.pos)
    xb = bits(x)
    _assert_partitions_equal(xb, p.pos, w.K, w.quant, recv, sc, w.R, w.S * w.K)
    _assert_combine_equal(xb, gates.reshape(w.T, w.K), w.K, w.quant, out, w.T)
    # properties that hold at any size, checked on the device as well
    pos_d = pb.pos.long()
    g_of_slot = torch.arange(w.N, device=dev()) // w.K
    if not w.quant:
        assert torch.equal(_row_checksum(recv)[pos_d], _row_checksum(x_d)[g_of_slot])
        # identity expert with softmax gates gives back the token (as values: -0 -> +0)
        assert torch.equal(out.float(), x_d.float())
    else:
        first = pos_d.view(w.T, w.K)[:, 0]
        cs = _row_checksum(recv)
        assert torch.equal(cs[pos_d].view(w.T, w.K), cs[first][:, None].expand(w.T, w.K))
        assert torch.equal(sc[pos_d].view(w.T, w.K), sc[first][:, None].expand(w.T, w.K))


def test_full_r8_combine_random_expert_rows():
    """Full-size combine on arbitrary expert rows (not copies of the token), every output
    against the oracle's combine over the oracle's plan."""
    w = synth.get("r8")
    ids, gates = synth.router(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    y = synth.expert_outputs(w, w.N)
    y_d = y.to(dev())
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(y_d, pb.pos, torch.from_numpy(gates).to(dev()), w.K, out)
    yb = bits(y)
    g = gates.reshape(w.T, w.K)
    pos = p.pos.reshape(w.T, w.K)
    chunk = 4096

    def one(t0):
        t1 = min(w.T, t0 + chunk)
        ref = oracle.combine(yb, pos[t0:t1], g[t0:t1], w.K)
        assert np.array_equal(bits(out[t0:t1]), ref), t0
        return t1 - t0
    with ThreadPoolExecutor(_POOL) as ex:
        assert sum(ex.map(one, range(0, w.T, chunk))) == w.T


def test_mapping_workload_dispatch_combine_exact():
    """The page-4 op end to end: mapping + pruning on every rank, grouped plan over the
    272 physical instances, dispatch H=4096, combine; every element compared."""
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    n_keys = w.R * w.place_per_rank
    for mode in (0, 1):
        bi = torch.empty((w.T, w.K), dtype=torch.int32, device=dev())
        bm = torch.empty((w.T, w.K), dtype=torch.uint8, device=dev())
        oi = np.empty_like(ids)
        om = np.empty(ids.shape, bool)
        for r in range(w.R):
            sl = slice(r * w.S, (r + 1) * w.S)
            mep.mep_update_expert(torch.from_numpy(ids[sl].copy()).to(dev()),
                                  torch.from_numpy(table).to(dev()),
                                  torch.from_numpy(gates[sl].copy()).to(dev()),
                                  torch.from_numpy(thr).to(dev()),
                                  torch.from_numpy(active[sl].astype(np.uint8)).to(dev()),
                                  r, w.R, mode, bi[sl], bm[sl])
            oi[sl], om[sl] = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, w.R, mode)
        pb = mep.PlanBuffers.allocate(w.R, n_keys, w.S, w.K, dev())
        mep.mep_plan(bi.view(-1), w.R, n_keys, w.S, w.K, pb, mode=mep.MEP_PLAN_GROUPED,
                     keys_per_rank=w.place_per_rank, keep=bm.view(-1))
        p = oracle.plan_grouped(oi, om, w.R, n_keys, w.place_per_rank, w.S, w.K)
        assert np.array_equal(pb.pos.cpu().numpy(), p.pos)
        x = synth.hidden(w)
        rows = p.n_kept
        recv = torch.zeros((rows, w.H), dtype=torch.bfloat16, device=dev())
        mep.mep_dispatch(x.to(dev()), pb.pos, w.K, recv)
        y_ref = oracle.dispatch(bits(x), p.pos, w.K, rows)
        assert np.array_equal(bits(recv), y_ref)
        out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
        mep.mep_combine(recv, pb.pos, torch.from_numpy(gates).to(dev()), w.K, out)
        assert np.array_equal(bits(out), oracle.combine(y_ref, p.pos, gates, w.K))
        # inactive tokens come back as zero rows
        inactive = np.flatnonzero(~active)
        assert not bits(out[torch.from_numpy(inactive).to(dev())]).any()
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("case", ["huge_row", "misaligned"])
def test_dispatch_fallback_paths(case):
    """Rows too large to stage twice in shared memory take the 16-byte register path;
    buffers that are not 16-byte aligned take the element path. Both must agree with
    the oracle like the staged path does."""
    rng = np.random.default_rng(31)
    if case == "huge_row":
        T, K, H = 6, 3, 51200
        x = _rand_bf16((T, H), 5)
        x_d = x.to(dev())
        rows = T * K
        recv = torch.zeros((rows, H), dtype=torch.bfloat16, device=dev())
    else:
        T, K, H = 9, 4, 64
        x = _rand_bf16((T, H), 6)
        flat = torch.zeros(T * H + 4, dtype=torch.bfloat16, device=dev())
        x_d = flat[4:].view(T, H)                      # 8 bytes off a 16-byte boundary
        x_d.copy_(x.to(dev()))
        rows = T * K
        rflat = torch.zeros(rows * H + 4, dtype=torch.bfloat16, device=dev())
        recv = rflat[4:].view(rows, H)
    pos = rng.permutation(rows).astype(np.int32)
    pos[rng.random(T * K) < 0.2] = -1
    pos_d = torch.from_numpy(pos).to(dev())
    mep.mep_dispatch(x_d, pos_d, K, recv)
    ref = oracle.dispatch(bits(x), pos, K, rows)
    assert np.array_equal(bits(recv), ref)
    gates = rng.random(T * K).astype(np.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(recv, pos_d, torch.from_numpy(gates).to(dev()), K, out)
    assert np.array_equal(bits(out), oracle.combine(ref, pos, gates, K))
    # the int8 dispatch on the same buffers (its fallbacks for large or unaligned rows)
    q = torch.zeros((rows, H), dtype=torch.int8, device=dev())
    q_view = q if case == "huge_row" else torch.zeros(rows * H + 8, dtype=torch.int8, device=dev())[8:].view(rows, H)
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    mep.mep_dispatch(x_d, pos_d, K, q_view, sc, quant=1)
    q_ref, s_ref = oracle.dispatch_int8(bits(x), pos, K, rows)
    assert np.array_equal(q_view.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("K", [1, 2, 3, 4, 6, 8, 16, 32])
@pytest.mark.parametrize("H", [8, 72, 4096, 7, 130])
def test_combine_int8_matches_oracle(K, H):
    """Combine of int8 rows with per-row scales (dequantisation in the sum): arbitrary
    codes, scales over several decades, dropped slots, every K, vector and element paths."""
    rng = np.random.default_rng(K * 1000 + H)
    T, rows = 61, 300
    q = rng.integers(-127, 128, (rows, H)).astype(np.int8)
    sc = (10.0 ** rng.uniform(-4, 2, rows)).astype(np.float32)
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.1] = -1
    gates = (rng.standard_normal(T * K)).astype(np.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine_int8(torch.from_numpy(q).to(dev()), torch.from_numpy(sc).to(dev()),
                         torch.from_numpy(pos).to(dev()), torch.from_numpy(gates).to(dev()), K, out)
    assert np.array_equal(bits(out), oracle.combine_int8(q, sc, pos, gates, K))
    assert mep.mep_get_error() == 0


def test_full_int8_workload_fused_combine():
    """The int8 workload end to end without bf16 rows, as bench.py runs it: plan, int8
    dispatch, combine of the int8 rows. Every output token against the oracle's dispatch,
    dequantisation and combine."""
    w = synth.get("int8")
    ids, gates = synth.router(w)
    x = synth.hidden(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    x_d = x.to(dev())
    g_d = torch.from_numpy(gates).to(dev())
    recv = torch.empty((w.N, w.H), dtype=torch.int8, device=dev())
    sc = torch.empty(w.N, dtype=torch.float32, device=dev())
    mep.mep_dispatch(x_d, pb.pos, w.K, recv, sc, quant=1)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine_int8(recv, sc, pb.pos, g_d, w.K, out)
    torch.cuda.synchronize()
    assert mep.mep_get_error() == 0
    _assert_combine_equal(bits(x), gates.reshape(w.T, w.K), w.K, 1, out, w.T)
