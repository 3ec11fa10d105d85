"""Seeded random shapes through the whole path on the GPU, every output compared whole
with the oracle: plan (all tables), dispatch (the whole receive buffer, bf16 or int8
codes and scales), combine (every output), and the dedup encoding with its round trip.
The shapes mix ragged and tiny sizes, odd hidden sizes (element paths), one rank, one
expert per rank, K up to 32 and heavy skew."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
from gpu_helpers import assert_plan_equal, bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu


def _case(seed):
    rng = np.random.default_rng(10_000 + seed)
    R = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
    per = int(rng.choice([1, 2, 3, 7, 8, 16, 64]))
    E = R * per
    K = int(rng.integers(1, min(E, 32) + 1))
    S = int(rng.integers(1, 300))
    H = int(rng.choice([8, 16, 24, 64, 200, 1024, 7, 13, 130, 777]))
    quant = int(rng.integers(0, 2))
    zipf = float(rng.choice([0.0, 1.0, 1.5, 3.0]))
    return rng, R, E, S, K, H, quant, zipf


@pytest.mark.parametrize("seed", range(100))
def test_fuzz_whole_path(seed):
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    rng, R, E, S, K, H, quant, zipf = _case(seed)
    T, N = R * S, R * S * K
    w = (np.arange(1, E + 1, dtype=np.float64) ** -zipf)[rng.permutation(E)]
    # distinct experts per token (top-K ids never repeat)
    ids = np.stack([rng.choice(E, K, replace=False, p=w / w.sum()) for _ in range(T)]).astype(np.int32).ravel()
    pb = gpu_plan_balanced(ids, R, E, S, K)
    p = oracle.plan_balanced(ids, R, E, S, K)
    assert_plan_equal(pb, p, R)

    x = torch.randn((T, H), generator=torch.Generator().manual_seed(seed)).mul(3).to(torch.bfloat16)
    xb = bits(x)
    z = rng.standard_normal((T, K))
    gates = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32).ravel()
    x_d, g_d = x.to(dev()), torch.from_numpy(gates).to(dev())
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    if quant:
        q = torch.zeros((N, H), dtype=torch.int8, device=dev())
        sc = torch.zeros(N, dtype=torch.float32, device=dev())
        mep.mep_dispatch(x_d, pb.pos, K, q, sc, quant=1)
        q_ref, s_ref = oracle.dispatch_int8(xb, p.pos, K, N)
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        mep.mep_combine_int8(q, sc, pb.pos, g_d, K, out)
        assert np.array_equal(bits(out), oracle.combine_int8(q_ref, s_ref, p.pos, gates, K))
    else:
        recv = torch.zeros((N, H), dtype=torch.bfloat16, device=dev())
        mep.mep_dispatch(x_d, pb.pos, K, recv)
        y_ref = oracle.dispatch(xb, p.pos, K, N)
        assert np.array_equal(bits(recv), y_ref)
        mep.mep_combine(recv, pb.pos, g_d, K, out)
        assert np.array_equal(bits(out), oracle.combine(y_ref, p.pos, gates, K))

    db = mep.DedupBuffers.allocate(R, S, K, dev())
    mep.mep_dedup_plan(pb.pos, pb.rank_off, R, S, K, db)
    d = oracle.dedup_plan(p.pos, K, p.rank_off)
    for name in ("dsend", "dpos", "drank_off", "dtok", "gidx"):
        assert np.array_equal(getattr(db, name).cpu().numpy(), getattr(d, name)), name
    U = int(d.drank_off[-1])
    sent = torch.empty((max(U, 1), H), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x_d, db.dsend, K, sent)
    back = torch.zeros((N, H), dtype=torch.bfloat16, device=dev())
    mep.mep_expand(sent, db.gidx, back)
    assert np.array_equal(bits(back), oracle.dispatch(xb, p.pos, K, N))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("seed", range(40))
def test_fuzz_mapping_grouped_path(seed):
    """Random eplb tables, both balance modes, pruning and active prefixes: the mapping of
    every rank in one launch, the grouped plan over the physical instances, then dispatch
    and combine with the dropped slots, all compared whole with the oracle."""
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    rng = np.random.default_rng(20_000 + seed)
    mode = int(rng.integers(0, 2))
    ws = int(rng.integers(2, 17))
    ppr = int(rng.integers(1, 40))
    n_keys = ws * ppr
    E = int(rng.integers(1, 300))
    K = int(rng.integers(1, min(16, E) + 1))
    F = int(rng.integers(2, min(ws + 1, 6) + 1))
    BS = int(rng.integers(1, 200))
    H = int(rng.choice([8, 64, 130, 256]))
    table = np.full((E, F), -1, np.int32)
    for e in range(E):
        c = int(rng.integers(1, F))
        table[e, 0] = c
        table[e, 1:1 + c] = rng.choice(n_keys, c, replace=False)
    T = ws * BS
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    sc = np.sort(rng.random((T, K)).astype(np.float32), axis=1)[:, ::-1].copy()
    thr = (rng.random(K) * 0.3).astype(np.float32)
    active = np.zeros(T, bool)
    for r in range(ws):
        active[r * BS: r * BS + int(rng.integers(0, BS + 1))] = True
    bi = torch.empty((T, K), dtype=torch.int32, device=dev())
    bm = torch.empty((T, K), dtype=torch.uint8, device=dev())
    mep.mep_update_expert_ranks(torch.from_numpy(ids).to(dev()), torch.from_numpy(table).to(dev()),
                                torch.from_numpy(sc).to(dev()), torch.from_numpy(thr).to(dev()),
                                torch.from_numpy(active.astype(np.uint8)).to(dev()), ws, mode, bi, bm)
    oi = np.empty_like(ids)
    om = np.empty(ids.shape, bool)
    for r in range(ws):
        sl = slice(r * BS, (r + 1) * BS)
        oi[sl], om[sl] = oracle.update_expert(ids[sl], table, sc[sl], thr, active[sl], r, ws, mode)
    assert np.array_equal(bi.cpu().numpy(), oi)
    assert np.array_equal(bm.cpu().numpy().astype(bool), om)

    pb = mep.PlanBuffers.allocate(ws, n_keys, BS, K, dev())
    mep.mep_plan(bi.view(-1), ws, n_keys, BS, K, pb, mode=mep.MEP_PLAN_GROUPED, keys_per_rank=ppr,
                 keep=bm.view(-1))
    p = oracle.plan_grouped(oi.ravel(), om.ravel(), ws, n_keys, ppr, BS, K)
    assert_plan_equal(pb, p, ws)

    N = T * K
    x = torch.randn((T, H), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    recv = torch.zeros((N, H), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x.to(dev()), pb.pos, K, recv)
    y_ref = oracle.dispatch(bits(x), p.pos, K, N)
    assert np.array_equal(bits(recv), y_ref)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    gates = sc.ravel()
    mep.mep_combine(recv, pb.pos, torch.from_numpy(gates).to(dev()), K, out)
    assert np.array_equal(bits(out), oracle.combine(y_ref, p.pos, gates, K))
    assert mep.mep_get_error() == 0
