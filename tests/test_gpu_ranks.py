"""Dispatch into, and combine from, the ranks' own receive buffers (mep_dispatch_ranks,
mep_combine_ranks) against the oracle.

Every EP rank's receive buffer is its own allocation, reached through a device table of
addresses (across GPUs these would be peer mappings; here they are separate buffers on
one GPU). Each source rank places its own slots with mep_plan_rank and dispatches its own
tokens; after all sources have, every rank's buffer must equal, bit for bit, the oracle's
dispatch restricted to that rank's partition of the global plan, and the combine read
back through the table must equal the oracle's combine."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def _route_by_ranks(w, quant):
    ids, gates = synth.router(w)
    x = synth.hidden(w)
    R, S, K, H, SK = w.R, w.S, w.K, w.H, w.S * w.K
    ids_r = ids.reshape(R, SK)
    hist_all = np.stack([oracle.histogram(ids_r[r], w.E) for r in range(R)]).astype(np.int32)
    hist_d = torch.from_numpy(hist_all).to(dev())
    dt = torch.int8 if quant else torch.bfloat16
    bufs = [torch.full((SK, H), 0x55 if quant else 0, dtype=dt, device=dev()) for _ in range(R)]
    scales = [torch.zeros(SK, dtype=torch.float32, device=dev()) for _ in range(R)] if quant else None
    table = mep.rank_pointer_table(bufs)
    stable = mep.rank_pointer_table(scales) if quant else None
    x_d = x.to(dev())
    rp = mep.RankPlanBuffers.allocate(R, w.E, S, K, dev())
    pos_all = np.empty(R * SK, np.int32)
    for src in range(R):                              # every source rank, one after another
        mep.mep_plan_rank(torch.from_numpy(ids_r[src].copy()).to(dev()), hist_d, R, w.E, S, K, src, rp)
        pos_all[src * SK:(src + 1) * SK] = rp.pos.cpu().numpy()
        mep.mep_dispatch_ranks(x_d[src * S:(src + 1) * S], rp.pos, K, table, SK, quant=quant, scale_table=stable)
    torch.cuda.synchronize()
    return ids, gates, x, bufs, scales, table, stable, pos_all


@pytest.mark.parametrize("name,quant", [("tiny", 0), ("tiny", 1), ("r8", 0), ("skew", 0), ("r8", 1)])
def test_dispatch_and_combine_through_rank_buffers(name, quant):
    w = synth.get(name)
    if name != "tiny":
        w = synth.scaled(w, S=512)                     # whole buffers against the oracle
    ids, gates, x, bufs, scales, table, stable, pos_all = _route_by_ranks(w, quant)
    SK = w.S * w.K
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    assert np.array_equal(pos_all, p.pos)
    xb = bits(x)
    for r in range(w.R):
        inside = (p.pos >= r * SK) & (p.pos < (r + 1) * SK)
        toks = np.unique(np.flatnonzero(inside) // w.K)
        pos_r = np.where(inside, p.pos - r * SK, -1).astype(np.int32).reshape(-1, w.K)[toks]
        if quant:
            q_ref, s_ref = oracle.dispatch_int8(xb[toks], pos_r, w.K, SK)
            assert np.array_equal(bufs[r].cpu().numpy(), q_ref), r
            assert np.array_equal(scales[r].cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), r
        else:
            assert np.array_equal(bits(bufs[r]), oracle.dispatch(xb[toks], pos_r, w.K, SK)), r
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine_ranks(table, torch.from_numpy(p.pos).to(dev()), torch.from_numpy(gates).to(dev()), w.K, SK, out,
                          quant=quant, scale_table=stable)
    pos_l = np.arange(w.N, dtype=np.int32)
    if quant:
        q, s = oracle.dispatch_int8(xb, pos_l, w.K, w.N)
        ref = oracle.combine_int8(q, s, pos_l, gates, w.K)
    else:
        ref = oracle.combine(oracle.dispatch(xb, pos_l, w.K, w.N), pos_l, gates, w.K)
    assert np.array_equal(bits(out), ref)
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("K", [1, 3, 8, 32])
@pytest.mark.parametrize("quant", [0, 1])
def test_rank_buffers_every_k_and_dropped_slots(K, quant):
    """Random rows and drops over 5 ranks of 40 rows each, every K path (compile-time and
    grouped runtime K), against the oracle over the concatenated buffers."""
    rng = np.random.default_rng(K * 10 + quant)
    R, rpr, T, H = 5, 40, 37, 64 if quant == 0 else 96
    n = T * K
    pos = rng.permutation(R * rpr)[:n].astype(np.int32) if n <= R * rpr else rng.integers(0, R * rpr, n).astype(np.int32)
    if n > R * rpr:
        pos = np.where(np.arange(n) < R * rpr, pos, -1).astype(np.int32)   # unique rows where kept
        pos[: R * rpr] = rng.permutation(R * rpr)
    pos[rng.random(n) < 0.2] = -1
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(K)) * 3).to(torch.bfloat16)
    dt = torch.int8 if quant else torch.bfloat16
    bufs = [torch.zeros((rpr, H), dtype=dt, device=dev()) for _ in range(R)]
    scales = [torch.zeros(rpr, dtype=torch.float32, device=dev()) for _ in range(R)] if quant else None
    table = mep.rank_pointer_table(bufs)
    stable = mep.rank_pointer_table(scales) if quant else None
    pos_d = torch.from_numpy(pos).to(dev())
    mep.mep_dispatch_ranks(x.to(dev()), pos_d, K, table, rpr, quant=quant, scale_table=stable)
    torch.cuda.synchronize()
    if quant:
        q_ref, s_ref = oracle.dispatch_int8(bits(x), pos, K, R * rpr)
        assert np.array_equal(torch.cat(bufs).cpu().numpy(), q_ref)
        assert np.array_equal(torch.cat(scales).cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    else:
        y_ref = oracle.dispatch(bits(x), pos, K, R * rpr)
        assert np.array_equal(bits(torch.cat(bufs)), y_ref)
    gates = rng.standard_normal(n).astype(np.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine_ranks(table, pos_d, torch.from_numpy(gates).to(dev()), K, rpr, out, quant=quant,
                          scale_table=stable)
    if quant:
        ref = oracle.combine_int8(q_ref, s_ref, pos, gates, K)
    else:
        ref = oracle.combine(y_ref, pos, gates, K)
    assert np.array_equal(bits(out), ref)
    assert mep.mep_get_error() == 0


def test_bad_rows_and_table_entries_are_skipped_and_flagged():
    R, rpr, T, K, H = 3, 8, 4, 2, 64
    x = torch.ones((T, H), dtype=torch.bfloat16, device=dev())
    bufs = [torch.zeros((rpr, H), dtype=torch.bfloat16, device=dev()) for _ in range(R)]
    table = mep.rank_pointer_table(bufs)
    pos = torch.tensor([0, 9, 17, 24, 3, -1, 30, 1], dtype=torch.int32, device=dev())   # 24, 30: past R*rpr
    mep.mep_dispatch_ranks(x, pos, K, table, rpr)
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE
    assert bufs[0][0].float().sum().item() == H and bufs[1][1].float().sum().item() == H
    bad = table.clone()
    bad[1] = 0                                         # no buffer for rank 1
    bad[2] = table[2] + 2                              # misaligned
    before = [b.clone() for b in bufs]
    mep.mep_dispatch_ranks(x, torch.tensor([10, 18, 0, 1, 2, 3, 4, 5], dtype=torch.int32, device=dev()), K, bad, rpr)
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE
    assert torch.equal(bufs[1], before[1]) and torch.equal(bufs[2], before[2])
