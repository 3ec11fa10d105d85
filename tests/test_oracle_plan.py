"""Pins for the oracle's histogram and placement plans (no GPU).

The oracle sorts a tuple list; the checks here come from elsewhere: a hand-worked
example, the MoonEP invariants (exactly S*K rows per rank, every slot on a replica of
its own expert, at most R-1 redundant replicas, maxvio 0 after planning), a
pairwise-comparison brute force over every id tensor of a tiny shape, and special
cases whose plan is known in closed form.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
import synth
from plan_checks import check_balanced_plan


def test_histogram_matches_bincount_and_sums_to_n():
    rng = np.random.default_rng(5)
    for E in (1, 3, 16, 257):
        ids = rng.integers(0, E, size=1000).astype(np.int32)
        h = oracle.histogram(ids, E)
        assert h.sum() == ids.size
        assert np.array_equal(h, np.bincount(ids, minlength=E))


def test_histogram_rejects_out_of_range():
    with pytest.raises(oracle.OracleError):
        oracle.histogram(np.array([0, 4], np.int32), 4)
    with pytest.raises(oracle.OracleError):
        oracle.histogram(np.array([-1], np.int32), 4)


def test_plan_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "plan_hand_r2_e4_s2_k2.json")))
    R, E, S, K = g["R"], g["E"], g["S"], g["K"]
    ex = g["expected"]
    p = oracle.plan_balanced(np.array(g["ids"], np.int32), R, E, S, K)
    assert p.hist.tolist() == ex["hist"]
    assert p.load.tolist() == ex["load"]
    assert p.max_load == ex["max_load"]
    assert p.maxvio_before(S, K) == ex["maxvio_before"]
    assert p.maxvio_after(S, K) == ex["maxvio_after"]
    assert p.pos.tolist() == ex["pos"]
    assert p.rep_count.tolist() == ex["rep_count"]
    for r in range(R):
        c = p.rep_count[r]
        assert p.rep_key[r][:c].tolist() == ex["rep_expert"][r]
        assert p.rep_cu[r][: c + 1].tolist() == ex["rep_cu"][r]
    assert p.redundant == ex["redundant"]
    assert p.prefetched == ex["prefetched"]


def _brute_pos(ids, R, E, S, K):
    """Row of slot n = number of slots that precede it in the (home, e, n) order,
    counted by comparing every pair."""
    ids = np.asarray(ids).ravel()
    per = E // R
    N = ids.size
    out = np.zeros(N, np.int64)
    for n in range(N):
        kn = (ids[n] // per, ids[n], n)
        out[n] = sum(1 for m in range(N) if (ids[m] // per, ids[m], m) < kn)
    return out


def test_plan_exhaustive_tiny():
    """Every id tensor of R=2, E=4, S=2, K=2 (4^8 inputs... sampled every 7th) and
    every one of R=2, E=4, S=1, K=2 and R=2, E=2, S=2, K=1."""
    cases = [(2, 4, 1, 2, 1), (2, 2, 2, 1, 1), (2, 4, 2, 2, 7)]
    for R, E, S, K, stride in cases:
        N = R * S * K
        for i, combo in enumerate(itertools.product(range(E), repeat=N)):
            if i % stride:
                continue
            ids = np.array(combo, np.int32)
            p = oracle.plan_balanced(ids, R, E, S, K)
            assert np.array_equal(p.pos, _brute_pos(ids, R, E, S, K)), combo
            check_balanced_plan(ids, R, E, S, K, p.pos, p.rep_count, p.rep_key, p.rep_cu,
                                p.redundant)
            assert p.max_chunk == S * K
            # home loads and replica counts from first principles
            per = E // R
            assert np.array_equal(p.load, np.bincount(ids // per, minlength=R))
            spans = {}
            for n in range(N):
                spans.setdefault(int(ids[n]), set()).add(int(p.pos[n]) // (S * K))
            assert p.redundant == sum(len(s) - 1 for s in spans.values())
            assert p.prefetched == sum(1 for e, s in spans.items() for r in s if r != e // per)


@pytest.mark.parametrize("R,E,S,K", [(4, 8, 8, 2), (3, 9, 5, 3), (4, 16, 8, 4), (8, 64, 6, 8)])
def test_plan_random_invariants_and_bruteforce(R, E, S, K):
    rng = np.random.default_rng(R * 1000 + E)
    for trial in range(6):
        w = rng.zipf(1.5, size=E).astype(np.float64)
        ids = rng.choice(E, size=R * S * K, p=w / w.sum()).astype(np.int32)
        p = oracle.plan_balanced(ids, R, E, S, K)
        check_balanced_plan(ids, R, E, S, K, p.pos, p.rep_count, p.rep_key, p.rep_cu, p.redundant)
        assert p.maxvio_after(S, K) == 0.0
        if R * S * K <= 256:
            assert np.array_equal(p.pos, _brute_pos(ids, R, E, S, K))


def test_plan_balanced_input_keeps_experts_home():
    """Every expert with exactly N/E slots: nothing moves, no replica, each rank's
    chunk is exactly its own home experts in order."""
    R, E, S, K = 4, 16, 8, 2
    N = R * S * K
    rng = np.random.default_rng(1)
    ids = rng.permutation(np.repeat(np.arange(E), N // E)).astype(np.int32)
    p = oracle.plan_balanced(ids, R, E, S, K)
    assert p.redundant == 0 and p.prefetched == 0
    assert p.max_load == S * K and p.maxvio_before(S, K) == 0.0
    per = E // R
    for r in range(R):
        assert p.rep_key[r][: p.rep_count[r]].tolist() == list(range(r * per, (r + 1) * per))


def test_plan_single_hot_expert_spans_every_rank():
    """All slots on one expert: it spans all R chunks, R-1 redundant replicas, all of
    them off its home rank; maxvio before = R-1."""
    R, E, S, K = 4, 8, 4, 2
    ids = np.full(R * S * K, 5, np.int32)
    p = oracle.plan_balanced(ids, R, E, S, K)
    assert p.redundant == R - 1
    assert p.prefetched == R - 1   # home(5) = 2; ranks 0, 1, 3 hold replicas
    assert p.maxvio_before(S, K) == R - 1
    assert np.array_equal(p.pos, np.arange(R * S * K))


@pytest.mark.parametrize("name", ["tiny", "skew"])
def test_plan_generated_workloads(name):
    w = synth.get(name)
    if name == "skew":
        w = synth.scaled(w, S=64)
    ids, _ = synth.router(w)
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    check_balanced_plan(ids, w.R, w.E, w.S, w.K, p.pos, p.rep_count, p.rep_key, p.rep_cu,
                        p.redundant)
    assert p.hist.sum() == w.N
    if w.force_expert0:
        assert p.hist[0] == w.T


def test_grouped_plan_packs_kept_slots_by_instance():
    R, kpr, S, K = 4, 3, 5, 2
    n_keys = R * kpr
    rng = np.random.default_rng(3)
    keys = rng.integers(0, n_keys, size=R * S * K).astype(np.int32)
    keep = rng.random(R * S * K) < 0.7
    p = oracle.plan_grouped(keys, keep, R, n_keys, kpr, S, K)
    kept = np.flatnonzero(keep)
    assert np.all(p.pos[~keep] == -1)
    assert np.array_equal(np.sort(p.pos[kept]), np.arange(kept.size))
    # rows ordered by (instance, slot index); ranks are contiguous blocks
    order = sorted(kept.tolist(), key=lambda n: (keys[n], n))
    assert [p.pos[n] for n in order] == list(range(kept.size))
    assert np.array_equal(np.diff(p.rank_off), np.bincount(keys[kept] // kpr, minlength=R))
    assert p.n_kept == kept.size
    for r in range(R):
        c = p.rep_count[r]
        ks = p.rep_key[r][:c]
        assert np.all(ks // kpr == r)
        assert np.array_equal(np.diff(p.rep_cu[r][: c + 1]),
                              np.bincount(keys[kept], minlength=n_keys)[ks])
