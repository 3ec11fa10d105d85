"""Pins for the oracle's logical->physical mapping and pruning (no GPU).

Checked against: hand-worked tables, the sample call printed in the aclnnMoeUpdateExpert
doc, the doc's argument rules, and properties that follow from them.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth


def test_mapping_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "update_expert_hand.json")))
    table = np.array(g["eplb_table"], np.int32)
    ids = np.array(g["expert_ids"], np.int32)
    for r, exp in g["expected_mode0_by_rank"].items():
        out, mask = oracle.update_expert(ids, table, None, None, None, int(r), g["world_size"], 0)
        assert out.tolist() == exp
        assert mask.all()
    out, _ = oracle.update_expert(ids, table, None, None, None, 0, g["world_size"], 1)
    assert out.tolist() == g["expected_mode1"]


def test_mapping_page_sample(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "update_expert_sample_p4.json")))
    E, F = g["moe_expert_num"], g["F"]
    table = np.array(g["eplb_table_data"][: E * F], np.int32).reshape(E, F)
    ids = np.tile(np.arange(g["K"], dtype=np.int32), (g["BS"], 1))
    for rank in range(g["world_size"]):
        out, mask = oracle.update_expert(ids, table, None, None, None, rank, g["world_size"],
                                         g["balance_mode"])
        assert out.tolist() == g["expected_ids_every_rank"]
        assert mask.all()


def test_mode0_column_never_exceeds_count():
    """With a true ceiling, local_rank / ceil(ws/c) + 1 <= c for every rank; a floor
    division would step past the instance list (e.g. ws=4, c=3, rank 3 -> column 4)."""
    for ws in range(2, 40):
        for c in range(2, min(ws, 15) + 1):
            F = c + 1
            table = np.array([[c] + list(range(10, 10 + c))], np.int32)
            seen = set()
            for rank in range(ws):
                out, _ = oracle.update_expert(np.zeros((1, 1), np.int32), table, None, None, None,
                                              rank, ws, 0)
                seen.add(int(out[0, 0]))
                assert 10 <= out[0, 0] < 10 + c
            # ranks are spread over a prefix of the instance list, at least 2 of them
            assert len(seen) >= 2 and seen == set(range(10, 10 + len(seen)))


def test_mode1_round_robin_by_token():
    table = np.array([[3, 7, 8, 9]], np.int32)
    ids = np.zeros((7, 1), np.int32)
    out, _ = oracle.update_expert(ids, table, None, None, None, 0, 4, 1)
    assert out[:, 0].tolist() == [7, 8, 9, 7, 8, 9, 7]


def test_pruning_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pruning_hand.json")))
    sc = np.array(g["expert_scales"], np.float32)
    thr = np.array(g["pruning_threshold"], np.float32)
    act = np.array(g["active_mask"], bool)
    ids = np.tile(np.arange(sc.shape[1], dtype=np.int32), (sc.shape[0], 1))
    table = np.array([[1, e] for e in range(sc.shape[1])], np.int32)
    _, mask = oracle.update_expert(ids, table, sc, thr, act, 0, 2, 0)
    assert mask.tolist() == g["expected_mask"]


def test_argument_rules():
    ids = np.zeros((2, 2), np.int32)
    table = np.array([[1, 0]], np.int32)
    sc = np.full((2, 2), 0.5, np.float32)
    thr = np.zeros(2, np.float32)
    act = np.array([True, True])
    bad = [
        dict(scales=sc, thr=None, act=None),                  # scales without threshold
        dict(scales=None, thr=thr, act=None),                 # threshold without scales
        dict(scales=None, thr=None, act=act),                 # mask without scales+threshold
    ]
    for b in bad:
        with pytest.raises(oracle.OracleError):
            oracle.update_expert(ids, table, b["scales"], b["thr"], b["act"], 0, 2, 0)
    with pytest.raises(oracle.OracleError):   # mask must have every True before every False
        oracle.update_expert(ids, table, sc, thr, np.array([False, True]), 0, 2, 0)
    with pytest.raises(oracle.OracleError):   # rank outside [0, world_size)
        oracle.update_expert(ids, table, None, None, None, 2, 2, 0)
    with pytest.raises(oracle.OracleError):   # world_size below 2 in mode 0
        oracle.update_expert(ids, table, None, None, None, 0, 1, 0)
    with pytest.raises(oracle.OracleError):   # expert id out of range
        oracle.update_expert(np.array([[1, 0]], np.int32), table, None, None, None, 0, 2, 0)
    with pytest.raises(oracle.OracleError):   # count 0 is not a valid instance count
        oracle.update_expert(ids, np.array([[0, 0]], np.int32), None, None, None, 0, 2, 0)
    with pytest.raises(oracle.OracleError):   # K > 16
        oracle.update_expert(np.zeros((1, 17), np.int32), np.zeros((32, 2), np.int32) + [1, 0],
                             None, None, None, 0, 2, 0)
    with pytest.raises(oracle.OracleError):   # balance_mode outside {0, 1}
        oracle.update_expert(ids, table, None, None, None, 0, 2, 2)


def test_generated_mapping_workload_properties():
    """On the page-4-shaped workload: every slot maps to an instance of its own expert,
    the top-1 slot of every active token survives pruning (threshold sum <= 0.1 <
    1/K <= top gate), kept slots form a prefix in k, and inactive tokens are dropped."""
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    inst_of = {}
    for e in range(w.E):
        for j in range(1, table[e, 0] + 1):
            inst_of[int(table[e, j])] = e
    assert sorted(inst_of) == list(range(w.R * w.place_per_rank))
    for mode in (0, 1):
        for r in range(w.R):
            sl = slice(r * w.S, (r + 1) * w.S)
            out, mask = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, w.R, mode)
            assert all(inst_of[int(i)] == int(e) for i, e in zip(out.ravel(), ids[sl].ravel()))
            act = active[sl]
            assert np.all(mask[act, 0])
            assert not mask[~act].any()
            # prefix property: once a slot is pruned every later slot is too
            assert np.all(np.diff(mask.astype(np.int8), axis=1) <= 0)


def test_grouped_receive_rows_within_the_setup_docs_bound():
    """The receive buffer bound of the aclnnMoeDistributeDispatchSetup doc (约束说明 5, A):
    a rank may receive at most BS * world_size * min(experts on the rank, K) token-slots,
    since every source rank sends BS tokens and a token's K distinct experts put at most
    min(local instances, K) of its slots on one rank. The grouped plan after the mapping
    keeps within it on the mapping workload in both modes, and under random tables with
    every token active and nothing pruned."""
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    n_keys = w.R * w.place_per_rank
    bound = w.S * w.R * min(w.place_per_rank, w.K)
    for mode in (0, 1):
        keys = np.empty_like(ids)
        keep = np.empty(ids.shape, bool)
        for r in range(w.R):
            sl = slice(r * w.S, (r + 1) * w.S)
            keys[sl], keep[sl] = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, w.R, mode)
        p = oracle.plan_grouped(keys.ravel(), keep.ravel(), w.R, n_keys, w.place_per_rank, w.S, w.K)
        assert np.diff(p.rank_off).max() <= bound
    rng = np.random.default_rng(11)
    for _ in range(20):
        ws, kpr, BS = int(rng.integers(2, 6)), int(rng.integers(1, 4)), int(rng.integers(1, 30))
        E = ws * kpr
        K = int(rng.integers(1, min(E, 8) + 1))
        # each expert one instance, a random permutation of the physical slots
        table = np.full((E, 2), -1, np.int32)
        table[:, 0] = 1
        table[:, 1] = rng.permutation(E)
        ids = np.stack([rng.choice(E, K, replace=False) for _ in range(ws * BS)]).astype(np.int32)
        keys = np.concatenate([oracle.update_expert(ids[r * BS:(r + 1) * BS], table, None, None, None, r, ws, 0)[0]
                               for r in range(ws)])
        p = oracle.plan_grouped(keys.ravel(), None, ws, E, kpr, BS, K)
        assert np.diff(p.rank_off).max() <= BS * ws * min(kpr, K)
