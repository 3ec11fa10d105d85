"""GPU parity of the deduplicated dispatch encoding (one row per token and destination
rank) and of the expansion on the receiving side, against the oracle on the same seeded
inputs (bit-exact), plus the round trip through dispatch at full workload sizes."""
import json
import os

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from dedup_checks import check_dedup
from gpu_helpers import bits, dev, gpu_plan_balanced, gpu_plan_grouped

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def gpu_dedup(pos, rank_off, R, S, K):
    db = mep.DedupBuffers.allocate(R, S, K, dev())
    p = pos if torch.is_tensor(pos) else torch.from_numpy(np.ascontiguousarray(pos, np.int32)).to(dev())
    ro = rank_off if torch.is_tensor(rank_off) else torch.from_numpy(np.ascontiguousarray(rank_off, np.int32)).to(dev())
    mep.mep_dedup_plan(p, ro, R, S, K, db)
    return db


def assert_dedup_equal(db, d):
    assert np.array_equal(db.dsend.cpu().numpy(), d.dsend), "dsend"
    assert np.array_equal(db.dpos.cpu().numpy(), d.dpos), "dpos"
    assert np.array_equal(db.drank_off.cpu().numpy(), d.drank_off), "drank_off"
    assert np.array_equal(db.dtok.cpu().numpy(), d.dtok), "dtok"
    assert np.array_equal(db.gidx.cpu().numpy(), d.gidx), "gidx"


def as_oracle(db):
    return oracle.Dedup(db.dsend.cpu().numpy(), db.dpos.cpu().numpy(), db.drank_off.cpu().numpy(),
                        db.dtok.cpu().numpy(), db.gidx.cpu().numpy())


def test_dedup_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "dedup_hand_r2_e4_s2_k2.json")))
    plan = json.load(open(os.path.join(golden_dir, "plan_hand_r2_e4_s2_k2.json")))
    db = gpu_dedup(np.array(plan["expected"]["pos"], np.int32), np.array(g["rank_off"], np.int32), 2, 2, g["K"])
    ex = g["expected"]
    U = ex["drank_off"][-1]
    assert db.dsend.cpu().tolist() == ex["dsend"]
    assert db.dpos.cpu().tolist() == ex["dpos"]
    assert db.drank_off.cpu().tolist() == ex["drank_off"]
    assert db.dtok.cpu().tolist()[:U] == ex["dtok"]
    assert db.gidx.cpu().tolist() == ex["gidx"]
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("R,E,S,K", [
    (2, 4, 3, 2), (4, 16, 37, 3), (8, 64, 300, 8), (1, 5, 17, 1), (3, 9, 1000, 1), (16, 4096, 32, 4),
    (5, 5, 2048, 5), (4, 64, 64, 32),
])
def test_dedup_parity_balanced(R, E, S, K):
    rng = np.random.default_rng(R * 7919 + E * 31 + S)
    w = rng.zipf(1.4, size=E).astype(np.float64)
    ids = rng.choice(E, size=R * S * K, p=w / w.sum()).astype(np.int32)
    pb = gpu_plan_balanced(ids, R, E, S, K)
    p = oracle.plan_balanced(ids, R, E, S, K)
    db = gpu_dedup(pb.pos, pb.rank_off, R, S, K)
    d = oracle.dedup_plan(p.pos, K, p.rank_off)
    assert_dedup_equal(db, d)
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("name", ["tiny", "r8", "skew"])
def test_dedup_parity_workloads(name):
    w = synth.get(name)
    ids, _ = synth.router(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    db = gpu_dedup(pb.pos, pb.rank_off, w.R, w.S, w.K)
    pos = pb.pos.cpu().numpy()
    rank_off = pb.rank_off.cpu().numpy()
    d = oracle.dedup_plan(pos, w.K, rank_off)
    assert_dedup_equal(db, d)
    check_dedup(pos, w.K, rank_off, as_oracle(db))
    assert mep.mep_get_error() == 0


def test_dedup_parity_grouped_plan_with_dropped_slots():
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    bi = torch.empty((w.T, w.K), dtype=torch.int32, device=dev())
    bm = torch.empty((w.T, w.K), dtype=torch.uint8, device=dev())
    mep.mep_update_expert_ranks(torch.from_numpy(ids).to(dev()), torch.from_numpy(table).to(dev()),
                                torch.from_numpy(gates).to(dev()), torch.from_numpy(thr).to(dev()),
                                torch.from_numpy(active.astype(np.uint8)).to(dev()), w.R, 0, bi, bm)
    n_keys = w.R * w.place_per_rank
    pb = gpu_plan_grouped(bi.cpu().numpy(), bm.cpu().numpy(), w.R, n_keys, w.place_per_rank, w.S, w.K)
    db = gpu_dedup(pb.pos, pb.rank_off, w.R, w.S, w.K)
    d = oracle.dedup_plan(pb.pos.cpu().numpy(), w.K, pb.rank_off.cpu().numpy())
    assert_dedup_equal(db, d)
    assert db.drank_off[-1].item() < pb.stats_dict()["n_kept"]
    assert mep.mep_get_error() == 0


def test_dedup_empty_ranks_and_all_dropped():
    """Ranks without rows (repeated offsets) and a plan whose slots are all dropped."""
    R, S, K = 4, 6, 3
    rng = np.random.default_rng(5)
    kept = 30
    pos = np.full(R * S * K, -1, np.int32)
    pos[rng.permutation(R * S * K)[:kept]] = np.arange(kept, dtype=np.int32)
    for rank_off in ([0, 0, 10, 10, 30], [0, 30, 30, 30, 30], [0, 7, 8, 29, 30]):
        ro = np.array(rank_off, np.int32)
        db = gpu_dedup(pos, ro, R, S, K)
        assert_dedup_equal(db, oracle.dedup_plan(pos, K, ro))
    none = np.full(R * S * K, -1, np.int32)
    ro = np.zeros(R + 1, np.int32)
    db = gpu_dedup(none, ro, R, S, K)
    assert_dedup_equal(db, oracle.dedup_plan(none, K, ro))
    assert mep.mep_get_error() == 0


def test_dedup_bad_rows_flag_and_drop():
    R, S, K = 2, 4, 2
    pos = np.arange(R * S * K, dtype=np.int32)
    pos[[3, 9]] = [R * S * K, -5]
    ro = np.array([0, 8, 16], np.int32)
    db = gpu_dedup(pos, ro, R, S, K)
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE
    dpos = db.dpos.cpu().numpy()
    assert dpos[3] == -1 and dpos[9] == -1
    clean = pos.copy()
    clean[[3, 9]] = -1
    assert_dedup_equal(db, oracle.dedup_plan(clean, K, ro))


@pytest.mark.parametrize("name", ["r8", "skew"])
def test_dedup_round_trip_full_workload(name):
    """Dispatch along the send list, expand on the receiving side: every row equals the
    plain dispatch's row (bit for bit, whole receive buffer)."""
    w = synth.get(name)
    ids, _ = synth.router(w)
    x = synth.hidden(w).to(dev())
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    db = gpu_dedup(pb.pos, pb.rank_off, w.R, w.S, w.K)
    U = int(db.drank_off[-1].item())
    sent = torch.empty((U, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x, db.dsend, w.K, sent)
    recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_expand(sent, db.gidx, recv)
    plain = torch.empty_like(recv)
    mep.mep_dispatch(x, pb.pos, w.K, plain)
    assert torch.equal(recv.view(torch.int16), plain.view(torch.int16))
    # the sent rows are the tokens' rows
    toks = db.dtok[:U].long()
    assert torch.equal(sent.view(torch.int16), x[toks].view(torch.int16))
    assert U < w.N
    assert mep.mep_get_error() == 0


def test_dedup_round_trip_int8():
    """The same round trip on int8 rows with their scales."""
    w = synth.get("tiny")
    ids, _ = synth.router(w)
    x = synth.hidden(w).to(dev())
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    db = gpu_dedup(pb.pos, pb.rank_off, w.R, w.S, w.K)
    U = int(db.drank_off[-1].item())
    sq = torch.empty((U, w.H), dtype=torch.int8, device=dev())
    ss = torch.empty(U, dtype=torch.float32, device=dev())
    mep.mep_dispatch(x, db.dsend, w.K, sq, ss, quant=1)
    q = torch.empty((w.N, w.H), dtype=torch.int8, device=dev())
    s = torch.empty(w.N, dtype=torch.float32, device=dev())
    mep.mep_expand(sq, db.gidx, q, src_scale=ss, dst_scale=s)
    q_ref, s_ref = oracle.dispatch_int8(bits(x), pb.pos.cpu().numpy(), w.K, w.N)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("H,quant,offset", [(8, 0, 0), (7, 0, 0), (130, 0, 2), (64, 1, 0), (33, 1, 0),
                                            (4096, 1, 3)])
def test_expand_matches_oracle(H, quant, offset):
    """Vector and byte paths, odd widths and unaligned buffers, rows left untouched."""
    rng = np.random.default_rng(H * 10 + quant)
    src_rows, rows = 50, 120
    if quant:
        src = rng.integers(-128, 128, (src_rows, H)).astype(np.int8)
        sc = rng.random(src_rows).astype(np.float32)
    else:
        src = rng.integers(0, 2**16, (src_rows, H)).astype(np.uint16)
        sc = None
    gidx = rng.integers(-1, src_rows, rows).astype(np.int32)
    tdt = torch.int8 if quant else torch.bfloat16
    npdt = np.int8 if quant else np.int16
    raw = torch.zeros(src_rows * H + offset, dtype=tdt, device=dev())
    src_d = raw[offset:].view(src_rows, H)
    src_d.copy_(torch.from_numpy(src.view(npdt)).to(dev()).view(tdt))
    fill = rng.integers(0, 100, (rows, H)).astype(npdt)
    dst = torch.from_numpy(fill).to(dev()).view(tdt).clone()
    if quant:
        ds = torch.full((rows,), 7.0, dtype=torch.float32, device=dev())
        mep.mep_expand(src_d, torch.from_numpy(gidx).to(dev()), dst, src_scale=torch.from_numpy(sc).to(dev()),
                       dst_scale=ds)
        ref, ref_s = oracle.expand(src, gidx, rows, src_scale=sc, dst=fill.view(np.int8),
                                   dst_scale=np.full(rows, 7.0, np.float32))
        assert np.array_equal(ds.cpu().numpy(), ref_s)
        assert np.array_equal(dst.cpu().numpy(), ref)
    else:
        mep.mep_expand(src_d, torch.from_numpy(gidx).to(dev()), dst)
        ref = oracle.expand(src, gidx, rows, dst=fill.view(np.uint16))
        assert np.array_equal(bits(dst), ref)
    assert mep.mep_get_error() == 0
    bad = torch.tensor([0, src_rows], dtype=torch.int32, device=dev())
    mep.mep_expand(src_d, bad, dst[:2].clone(), src_scale=None if not quant else torch.from_numpy(sc).to(dev()),
                   dst_scale=None if not quant else torch.zeros(2, device=dev()))
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE
