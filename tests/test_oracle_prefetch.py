"""Pins for the oracle's replica weight prefetch and replica gradient reduce: a
hand-worked case, the properties every placement must have, exact conservation of
integer-valued gradients, and a case where the order of the fp32 additions matters."""
import json
import os

import numpy as np
import pytest

import oracle
import synth


def test_prefetch_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "prefetch_hand_r2_e4.json")))
    for c in g["cases"]:
        se, rw = oracle.prefetch_plan(np.array(g["rep_count"]), np.array(g["rep_key"]), g["R"], g["E"], c["B"])
        assert se.tolist() == c["slot_expert"]
        assert rw.tolist() == c["rep_weight"]


@pytest.mark.parametrize("name,B", [("r8", 8), ("r8", 3), ("skew", 8), ("skew", 1), ("tiny", 4)])
def test_prefetch_properties(name, B):
    w = synth.get(name)
    if name == "skew":
        w = synth.scaled(w, S=128)
    ids, _ = synth.router(w)
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    se, rw = oracle.prefetch_plan(p.rep_count, p.rep_key, w.R, w.E, B)
    per = w.E // w.R
    D = 6
    w_home = np.random.default_rng(0).integers(0, 2**16, (w.E, D)).astype(np.uint16)
    w_slots = oracle.prefetch_weights(w_home, se, w.R, B)
    allw = np.concatenate([w_home, w_slots.reshape(w.R * B, D)])
    prefetched = 0
    for r in range(w.R):
        keys = p.rep_key[r, : p.rep_count[r]]
        remote = [e for e in keys if e // per != r]
        used = int((se[r] >= 0).sum())
        assert used == min(B, len(remote))
        assert se[r, :used].tolist() == remote[:used]         # slots in replica order
        for j, e in enumerate(keys):
            assert np.array_equal(allw[rw[r, j]], w_home[e])  # every replica reads its expert
            if e // per == r:
                assert rw[r, j] == e                            # home replicas read home
        prefetched += len(remote)
    assert prefetched == p.prefetched


def test_grad_reduce_conserves_integer_gradients():
    rng = np.random.default_rng(1)
    E, R, B, D = 8, 4, 3, 50
    se = np.full((R, B), -1, np.int32)
    se[0, :2] = [5, 6]
    se[1, 0] = 5
    se[3, :3] = [0, 5, 7]
    gh = rng.integers(-1000, 1000, (E, D)).astype(np.float32)
    gs = rng.integers(-1000, 1000, (R * B, D)).astype(np.float32)
    nh, ns = oracle.grad_reduce(gh, gs, se, R, B)
    flat = se.ravel()
    for e in range(E):
        want = gh[e] + gs[flat == e].sum(0)
        assert np.array_equal(nh[e], want)
    assert not ns[flat >= 0].any()
    assert np.array_equal(ns[flat < 0], gs[flat < 0])           # unused slots untouched


def test_grad_reduce_adds_in_ascending_rank_order():
    """1 + 2^24 + 1 in fp32: rank 0's 2^24 first gives 2^24, rank 1's first gives 2^24+2."""
    E, R, B, D = 2, 2, 1, 1
    se = np.array([[1], [1]], np.int32)
    gh = np.array([[0.0], [1.0]], np.float32)
    gs = np.array([[2.0 ** 24], [1.0]], np.float32)
    nh, _ = oracle.grad_reduce(gh, gs, se, R, B)
    assert nh[1, 0] == np.float32(2.0 ** 24)
    gs2 = np.array([[1.0], [2.0 ** 24]], np.float32)
    nh2, _ = oracle.grad_reduce(gh, gs2, se, R, B)
    assert nh2[1, 0] == np.float32(2.0 ** 24 + 2.0)
