"""GPU parity of the histogram, balanced and grouped plans, and the mapping op,
against the oracle on the same seeded inputs (bit-exact)."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import assert_plan_equal, dev, gpu_plan_balanced, gpu_plan_grouped
from plan_checks import check_balanced_plan
from dedup_checks import check_dedup

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def test_histogram_parity_ragged_and_skewed():
    rng = np.random.default_rng(0)
    for n, E in [(0, 4), (1, 1), (2047, 16), (2049, 64), (100_003, 512), (1 << 20, 4096)]:
        ids = rng.zipf(1.3, size=n).astype(np.int64) % E
        ids = ids.astype(np.int32)
        h = torch.empty(E, dtype=torch.int32, device=dev())
        mep.mep_histogram(torch.from_numpy(ids).to(dev()), E, h)
        assert np.array_equal(h.cpu().numpy(), oracle.histogram(ids, E))
    assert mep.mep_get_error() == 0


# Plans of at most 16384 slots run in one launch: over a cluster of 8 CTAs when at most
# 1421 keys fit its shared memory, else in one CTA (up to 1504 keys); the others as the
# tiled four-kernel sort (tiles of 512, 1024 or 2048 slots by size). The cases cover each
# path, at and just past the boundaries (ragged last tiles and CTA shares), and small
# plans whose keys are too many for either one-launch path.
@pytest.mark.parametrize("R,E,S,K", [
    (2, 4, 2, 2), (3, 9, 37, 3), (4, 12, 1000, 3), (4, 16, 128, 2), (8, 64, 300, 8),
    (1, 5, 17, 1), (16, 4096, 32, 4), (8, 4096, 512, 8), (5, 5, 2048, 1),
    (4, 16, 1024, 4), (7, 7, 2340, 1), (2, 1024, 4096, 2), (3, 9, 1821, 3), (1, 2, 16385, 1),
    (64, 1536, 8, 8),
    # the cluster at its key limit, the one-CTA plan past it, both at 16384 slots
    (8, 1416, 256, 8), (8, 1480, 256, 8), (4, 1420, 1024, 4),
    # CTA shares that end inside a warp's range, and CTAs left without slots
    (1, 3, 8191, 2), (1, 3, 33, 1), (3, 6, 5, 7),
    # ragged last tiles of the 1024- and 2048-slot tiles (more than 2^18 and 2^20 slots)
    (7, 7, 37454, 1), (5, 10, 209916, 1),
])
def test_plan_balanced_parity_random(R, E, S, K):
    rng = np.random.default_rng(R * 7919 + E * 31 + S)
    w = rng.zipf(1.4, size=E).astype(np.float64)
    ids = rng.choice(E, size=R * S * K, p=w / w.sum()).astype(np.int32)
    pb = gpu_plan_balanced(ids, R, E, S, K)
    p = oracle.plan_balanced(ids, R, E, S, K)
    assert_plan_equal(pb, p, R)
    assert mep.mep_get_error() == 0


def test_plan_balanced_single_expert_and_uniform():
    R, E, S, K = 8, 16, 512, 4
    for ids in [np.full(R * S * K, 3, np.int32),
                np.random.default_rng(2).permutation(np.repeat(np.arange(E), R * S * K // E)).astype(np.int32)]:
        pb = gpu_plan_balanced(ids, R, E, S, K)
        assert_plan_equal(pb, oracle.plan_balanced(ids, R, E, S, K), R)


@pytest.mark.parametrize("name", ["tiny", "r8", "int8", "skew"])
def test_plan_balanced_parity_workloads(name):
    """Full-size workloads: the whole plan, bit for bit, plus the MoonEP invariants."""
    w = synth.get(name)
    ids, _ = synth.router(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    assert_plan_equal(pb, p, w.R)
    check_balanced_plan(ids, w.R, w.E, w.S, w.K, pb.pos.cpu().numpy(), pb.rep_count.cpu().numpy(),
                        pb.rep_key.cpu().numpy(), pb.rep_cu.cpu().numpy(),
                        pb.stats_dict()["redundant"])
    assert pb.stats_dict()["max_chunk"] == w.S * w.K
    assert mep.mep_get_error() == 0


def test_plan_out_of_range_ids_flag_and_drop():
    R, E, S, K = 2, 4, 64, 2
    ids = np.random.default_rng(3).integers(0, E, R * S * K).astype(np.int32)
    ids[[5, 77]] = [E, -3]
    pb = gpu_plan_balanced(ids, R, E, S, K)
    assert mep.mep_get_error() & mep.DERR_KEY_RANGE
    pos = pb.pos.cpu().numpy()
    assert pos[5] == -1 and pos[77] == -1
    assert mep.mep_get_error() == 0   # cleared by the previous read


def _mapping_all_ranks(w, mode, gpu: bool):
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    out_ids = np.empty_like(ids)
    out_mask = np.empty(ids.shape, bool)
    for r in range(w.R):
        sl = slice(r * w.S, (r + 1) * w.S)
        if gpu:
            bi = torch.empty((w.S, w.K), dtype=torch.int32, device=dev())
            bm = torch.empty((w.S, w.K), dtype=torch.uint8, device=dev())
            mep.mep_update_expert(torch.from_numpy(ids[sl].copy()).to(dev()),
                                  torch.from_numpy(table).to(dev()),
                                  torch.from_numpy(gates[sl].copy()).to(dev()),
                                  torch.from_numpy(thr).to(dev()),
                                  torch.from_numpy(active[sl].astype(np.uint8)).to(dev()),
                                  r, w.R, mode, bi, bm)
            out_ids[sl] = bi.cpu().numpy()
            out_mask[sl] = bm.cpu().numpy().astype(bool)
        else:
            o, m = oracle.update_expert(ids[sl], table, gates[sl], thr, active[sl], r, w.R, mode)
            out_ids[sl] = o
            out_mask[sl] = m
    return ids, gates, out_ids, out_mask


@pytest.mark.parametrize("mode", [0, 1])
def test_update_expert_and_grouped_plan_parity(mode):
    w = synth.get("map")
    _, _, gi, gm = _mapping_all_ranks(w, mode, gpu=True)
    _, _, oi, om = _mapping_all_ranks(w, mode, gpu=False)
    assert np.array_equal(gi, oi) and np.array_equal(gm, om)
    assert mep.mep_get_error() == 0
    n_keys = w.R * w.place_per_rank
    pb = gpu_plan_grouped(gi, gm, w.R, n_keys, w.place_per_rank, w.S, w.K)
    p = oracle.plan_grouped(oi, om, w.R, n_keys, w.place_per_rank, w.S, w.K)
    assert_plan_equal(pb, p, w.R)


@pytest.mark.parametrize("mode", [0, 1])
def test_update_expert_ranks_matches_per_rank_oracle(mode):
    """One launch over every rank's block equals the oracle called rank by rank."""
    w = synth.get("map")
    ids, gates = synth.router(w)
    table, thr, active = synth.mapping_inputs(w)
    bi = torch.empty((w.T, w.K), dtype=torch.int32, device=dev())
    bm = torch.empty((w.T, w.K), dtype=torch.uint8, device=dev())
    mep.mep_update_expert_ranks(torch.from_numpy(ids).to(dev()), torch.from_numpy(table).to(dev()),
                                torch.from_numpy(gates).to(dev()), torch.from_numpy(thr).to(dev()),
                                torch.from_numpy(active.astype(np.uint8)).to(dev()), w.R, mode, bi, bm)
    _, _, oi, om = _mapping_all_ranks(w, mode, gpu=False)
    assert np.array_equal(bi.cpu().numpy(), oi) and np.array_equal(bm.cpu().numpy().astype(bool), om)
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("ws,BS,K,E,F", [(2, 1, 1, 1, 2), (3, 37, 3, 9, 3), (7, 129, 4, 16, 5)])
def test_update_expert_ranks_ragged_no_pruning(ws, BS, K, E, F):
    """Ragged block sizes, no scales: every slot is mapped and kept."""
    rng = np.random.default_rng(ws * 100 + BS)
    ids = np.stack([rng.permutation(E)[:K] for _ in range(ws * BS)]).astype(np.int32)
    table = np.zeros((E, F), np.int32)
    for e in range(E):
        c = int(rng.integers(1, F))
        table[e, 0] = c
        table[e, 1:1 + c] = rng.integers(0, ws * 4, c)
    for mode in (0, 1) if ws >= 2 else (1,):
        bi = torch.empty((ws * BS, K), dtype=torch.int32, device=dev())
        bm = torch.empty((ws * BS, K), dtype=torch.uint8, device=dev())
        mep.mep_update_expert_ranks(torch.from_numpy(ids).to(dev()), torch.from_numpy(table).to(dev()),
                                    None, None, None, ws, mode, bi, bm)
        for r in range(ws):
            sl = slice(r * BS, (r + 1) * BS)
            o, m = oracle.update_expert(ids[sl], table, None, None, None, r, ws, mode)
            assert np.array_equal(bi.cpu().numpy()[sl], o)
            assert np.array_equal(bm.cpu().numpy()[sl].astype(bool), m)
    assert mep.mep_get_error() == 0


def test_update_expert_ranks_mask_is_per_rank_block():
    """A 0 then 1 across a rank boundary is allowed; inside one rank's block it is flagged."""
    ids = torch.tensor([[0, 1], [1, 0], [0, 1], [1, 0]], dtype=torch.int32, device=dev())
    table = torch.tensor([[1, 0, 0], [2, 1, 0]], dtype=torch.int32, device=dev())
    sc = torch.full((4, 2), 0.5, dtype=torch.float32, device=dev())
    thr = torch.zeros(2, dtype=torch.float32, device=dev())
    bi = torch.empty_like(ids)
    bm = torch.empty((4, 2), dtype=torch.uint8, device=dev())
    mep.mep_update_expert_ranks(ids, table, sc, thr, torch.tensor([1, 0, 1, 1], dtype=torch.uint8,
                                                                    device=dev()), 2, 0, bi, bm)
    assert mep.mep_get_error() == 0
    assert bm.cpu().tolist() == [[1, 1], [0, 0], [1, 1], [1, 1]]
    mep.mep_update_expert_ranks(ids, table, sc, thr, torch.tensor([1, 1, 0, 1], dtype=torch.uint8,
                                                                    device=dev()), 2, 0, bi, bm)
    assert mep.mep_get_error() & mep.DERR_MASK


def test_update_expert_hand_tables(golden_dir):
    import json, os
    g = json.load(open(os.path.join(golden_dir, "update_expert_hand.json")))
    table = torch.tensor(g["eplb_table"], dtype=torch.int32, device=dev())
    ids = torch.tensor(g["expert_ids"], dtype=torch.int32, device=dev())
    bi = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device=dev())
    for r, exp in g["expected_mode0_by_rank"].items():
        mep.mep_update_expert(ids, table, None, None, None, int(r), g["world_size"], 0, bi, bm)
        assert bi.cpu().tolist() == exp and bool(bm.all())
    mep.mep_update_expert(ids, table, None, None, None, 0, g["world_size"], 1, bi, bm)
    assert bi.cpu().tolist() == g["expected_mode1"]


def test_update_expert_data_errors_flag():
    ids = torch.tensor([[0, 1], [1, 0]], dtype=torch.int32, device=dev())
    bi = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device=dev())
    bad_table = torch.tensor([[0, 5], [1, 1]], dtype=torch.int32, device=dev())   # count 0
    mep.mep_update_expert(ids, bad_table, None, None, None, 0, 2, 0, bi, bm)
    assert mep.mep_get_error() & mep.DERR_TABLE
    assert bi.cpu().tolist() == [[-1, 1], [1, -1]]
    table = torch.tensor([[1, 0], [1, 1]], dtype=torch.int32, device=dev())
    sc = torch.full((2, 2), 0.5, dtype=torch.float32, device=dev())
    thr = torch.zeros(2, dtype=torch.float32, device=dev())
    mask = torch.tensor([0, 1], dtype=torch.uint8, device=dev())
    mep.mep_update_expert(ids, table, sc, thr, mask, 0, 2, 0, bi, bm)
    assert mep.mep_get_error() & mep.DERR_MASK
    oob = torch.tensor([[0, 7], [1, 0]], dtype=torch.int32, device=dev())
    mep.mep_update_expert(oob, table, None, None, None, 0, 2, 0, bi, bm)
    assert mep.mep_get_error() & mep.DERR_KEY_RANGE


@pytest.mark.parametrize("R,kpr,S,K", [(4, 5, 333, 3), (4, 34, 3000, 3), (8, 34, 256, 8)])
def test_grouped_plan_all_dropped_and_ragged(R, kpr, S, K):
    """One-CTA plans (the first and last shapes) and a tiled one (36,000 slots)."""
    rng = np.random.default_rng(9 + S)
    keys = rng.integers(0, R * kpr, R * S * K).astype(np.int32)
    for keep in [np.zeros(R * S * K, np.uint8), (rng.random(R * S * K) < 0.5).astype(np.uint8),
                 np.ones(R * S * K, np.uint8)]:
        pb = gpu_plan_grouped(keys, keep, R, R * kpr, kpr, S, K)
        assert_plan_equal(pb, oracle.plan_grouped(keys, keep, R, R * kpr, kpr, S, K), R)


def test_plan_and_dedup_at_the_largest_rank_and_key_counts():
    """R = n_keys = MEP_MAX_KEYS (4096 ranks of one expert each): the plan and its replica
    tables bit for bit against the oracle, the dedup encoding against every property an
    encoding of that plan must have (the oracle's rank-by-rank construction is too slow at
    4096 ranks); and one rank past the limit is refused."""
    R = E = 4096
    S, K = 2, 2
    rng = np.random.default_rng(4096)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(R * S)]).astype(np.int32).ravel()
    pb = gpu_plan_balanced(ids, R, E, S, K)
    p = oracle.plan_balanced(ids, R, E, S, K)
    assert_plan_equal(pb, p, R)
    db = mep.DedupBuffers.allocate(R, S, K, dev())
    mep.mep_dedup_plan(pb.pos, pb.rank_off, R, S, K, db)
    check_dedup(p.pos, K, p.rank_off, oracle.Dedup(*[getattr(db, n).cpu().numpy() for n in
                                                     ("dsend", "dpos", "drank_off", "dtok", "gidx")]))
    assert mep.mep_get_error() == 0
    with pytest.raises(mep.MepError) as e:
        mep.mep_plan(torch.zeros((R + 1) * S * K, dtype=torch.int32, device=dev()), R + 1, E + 1, S, K,
                     mep.PlanBuffers.allocate(R + 1, E + 1, S, K, dev()))
    assert e.value.status == 3
