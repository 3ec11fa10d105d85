"""Pins for the oracle's deduplicated dispatch encoding and its expansion (no GPU).

Checked against a hand-worked example, a count of distinct (token, rank) pairs taken
with numpy, the round trip through the already pinned dispatch (dispatching one row per
pair and expanding on the receiving side gives the plain dispatch's rows), the bounds a
dedup encoding must respect, and the special cases K = 1 and R = 1.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from dedup_checks import check_dedup


def test_dedup_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "dedup_hand_r2_e4_s2_k2.json")))
    plan = json.load(open(os.path.join(golden_dir, "plan_hand_r2_e4_s2_k2.json")))
    pos = np.array(plan["expected"]["pos"], np.int32)
    d = oracle.dedup_plan(pos, g["K"], np.array(g["rank_off"], np.int32))
    ex = g["expected"]
    U = ex["drank_off"][-1]
    assert d.dsend.tolist() == ex["dsend"]
    assert d.dpos.tolist() == ex["dpos"]
    assert d.drank_off.tolist() == ex["drank_off"]
    assert d.dtok[:U].tolist() == ex["dtok"]
    assert d.gidx.tolist() == ex["gidx"]


def _round_trip(x, pos, K, rank_off, d):
    rows = int(rank_off[-1])
    plain = oracle.dispatch(x, pos, K, max(rows, 1))
    U = int(d.drank_off[-1])
    sent = oracle.dispatch(x, d.dsend, K, max(U, 1))
    back = oracle.expand(sent, d.gidx, max(rows, 1))
    assert np.array_equal(back, plain)


@pytest.mark.parametrize("R,E,S,K", [(2, 4, 3, 2), (4, 16, 37, 3), (8, 64, 64, 8), (3, 3, 5, 3)])
def test_dedup_balanced_plans(R, E, S, K):
    rng = np.random.default_rng(R * 100 + S)
    w = rng.zipf(1.3, E).astype(float)
    ids = np.stack([rng.choice(E, K, replace=False, p=w / w.sum()) for _ in range(R * S)]).astype(np.int32)
    p = oracle.plan_balanced(ids.ravel(), R, E, S, K)
    rank_off = np.arange(R + 1, dtype=np.int32) * S * K
    d = oracle.dedup_plan(p.pos, K, rank_off)
    check_dedup(p.pos, K, rank_off, d)
    x = rng.integers(0, 2**16, (R * S, 9)).astype(np.uint16)
    _round_trip(x, p.pos, K, rank_off, d)


def test_dedup_grouped_plan_with_dropped_slots():
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    bi = np.empty_like(ids)
    bm = np.empty(ids.shape, bool)
    for r in range(w.R):
        sl = slice(r * w.S, (r + 1) * w.S)
        bi[sl], bm[sl] = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, w.R, 0)
    n_keys = w.R * w.place_per_rank
    p = oracle.plan_grouped(bi.ravel(), bm.ravel(), w.R, n_keys, w.place_per_rank, w.S, w.K)
    d = oracle.dedup_plan(p.pos, w.K, p.rank_off)
    check_dedup(p.pos, w.K, p.rank_off, d)
    assert d.drank_off[-1] < (p.pos >= 0).sum()           # some tokens hit a rank twice
    x = np.random.default_rng(1).integers(0, 2**16, (w.T, 16)).astype(np.uint16)
    _round_trip(x, p.pos, w.K, p.rank_off, d)


def test_dedup_k1_keeps_every_slot():
    rng = np.random.default_rng(2)
    R, S = 4, 50
    pos = rng.permutation(R * S).astype(np.int32)
    pos[rng.random(R * S) < 0.2] = -1
    kept = np.sort(pos[pos >= 0])
    # pack the kept rows (a grouped-style plan with dropped slots)
    remap = np.full(R * S, -1, np.int32)
    remap[kept] = np.arange(kept.size)
    pos = np.where(pos >= 0, remap[np.maximum(pos, 0)], -1).astype(np.int32)
    rank_off = np.linspace(0, kept.size, R + 1).astype(np.int32)
    d = oracle.dedup_plan(pos, 1, rank_off)
    check_dedup(pos, 1, rank_off, d)
    assert d.drank_off[-1] == kept.size
    assert np.array_equal(d.dsend, d.dpos)


def test_dedup_single_rank_sends_each_token_once():
    rng = np.random.default_rng(3)
    S, K = 40, 4
    pos = rng.permutation(S * K).astype(np.int32)
    pos[rng.random(S * K) < 0.3] = -1
    remap = np.full(S * K, -1, np.int32)
    kept = np.sort(pos[pos >= 0])
    remap[kept] = np.arange(kept.size)
    pos = np.where(pos >= 0, remap[np.maximum(pos, 0)], -1).astype(np.int32)
    d = oracle.dedup_plan(pos, K, np.array([0, kept.size], np.int32))
    tokens = np.unique(np.nonzero(pos >= 0)[0] // K)
    assert d.drank_off.tolist() == [0, tokens.size]
    assert np.array_equal(d.dtok[:tokens.size], tokens)


def test_dedup_rejects_bad_rows():
    with pytest.raises(oracle.OracleError):
        oracle.dedup_plan(np.array([0, 4], np.int32), 2, np.array([0, 2, 4], np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.dedup_plan(np.array([0, -2], np.int32), 2, np.array([0, 2, 4], np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.dedup_plan(np.array([0, 1], np.int32), 2, np.array([0, 3, 2], np.int32))


def test_expand_copies_rows_and_scales():
    rng = np.random.default_rng(4)
    src = rng.integers(-128, 128, (5, 7)).astype(np.int8)
    sc = rng.random(5).astype(np.float32)
    gidx = np.array([4, -1, 0, 0, 2, -1], np.int32)
    q, s = oracle.expand(src, gidx, 6, src_scale=sc)
    for p, u in enumerate(gidx):
        if u >= 0:
            assert np.array_equal(q[p], src[u]) and s[p] == sc[u]
        else:
            assert not q[p].any() and s[p] == 0
    with pytest.raises(oracle.OracleError):
        oracle.expand(src, np.array([5], np.int32), 1)
