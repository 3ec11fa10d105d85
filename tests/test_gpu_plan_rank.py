"""One EP rank's share of the balanced plan (mep_plan_rank) against the oracle.

Every rank of a workload is planned on its own, from its own ids and the per-rank
histograms of all ranks (the all-gathered matrix, here drawn from the oracle's
histogram of each rank's ids). The rows it gives each of its slots must be, bit for
bit, the rows of the oracle's plan over all ranks' ids (and of mep_plan on the GPU);
its send and receive counts must be the oracle plan's counts of rows crossing from
each source rank to each destination rank."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def _check_all_ranks(ids, R, E, S, K):
    ids = np.ascontiguousarray(ids, np.int32).reshape(R, S * K)
    p = oracle.plan_balanced(ids.ravel(), R, E, S, K)
    hist_all = np.stack([oracle.histogram(ids[r], E) for r in range(R)]).astype(np.int32)
    hist_d = torch.from_numpy(hist_all).to(dev())
    SK = S * K
    dest = p.pos.reshape(R, SK) // SK                  # destination rank of every slot
    # rows crossing from source s to destination d, counted on the oracle's plan
    cross = np.zeros((R, R), np.int64)
    np.add.at(cross, (np.repeat(np.arange(R), SK), dest.ravel()), 1)
    pb = gpu_plan_balanced(ids, R, E, S, K)
    gpu_pos = pb.pos.cpu().numpy().reshape(R, SK)
    out = mep.RankPlanBuffers.allocate(R, E, S, K, dev())
    for r in range(R):
        mep.mep_plan_rank(torch.from_numpy(ids[r].copy()).to(dev()), hist_d, R, E, S, K, r, out)
        pos = out.pos.cpu().numpy()
        assert np.array_equal(pos, p.pos.reshape(R, SK)[r]), r
        assert np.array_equal(pos, gpu_pos[r]), r
        sc, so = out.send_count.cpu().numpy(), out.send_off.cpu().numpy()
        rc, ro = out.recv_count.cpu().numpy(), out.recv_off.cpu().numpy()
        assert np.array_equal(sc, cross[r]), r
        assert np.array_equal(rc, cross[:, r]), r
        assert np.array_equal(so, np.concatenate([[0], np.cumsum(cross[r])])), r
        assert np.array_equal(ro, np.concatenate([[0], np.cumsum(cross[:, r])])), r
        assert ro[-1] == SK and so[-1] == SK
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("name", ["tiny", "r8", "skew"])
def test_every_rank_of_a_workload(name):
    w = synth.get(name)
    ids, _ = synth.router(w)
    _check_all_ranks(ids, w.R, w.E, w.S, w.K)


@pytest.mark.parametrize("R,E,S,K,s", [(1, 4, 300, 3, 0.0), (3, 9, 777, 5, 1.3), (7, 7, 2049, 1, 2.5),
                                       (16, 64, 129, 8, 0.8), (5, 40, 1000, 32, 1.1)])
def test_random_shapes(R, E, S, K, s):
    rng = np.random.default_rng(R * 100 + E + S)
    w = (np.arange(E) + 1.0) ** -s
    ids = rng.choice(E, size=R * S * K, p=w / w.sum()).astype(np.int32)   # repeats allowed
    _check_all_ranks(ids, R, E, S, K)


def test_disagreeing_histograms_are_flagged():
    w = synth.scaled(synth.get("tiny"), S=64)
    ids, _ = synth.router(w)
    ids = ids.reshape(w.R, -1)
    hist_all = np.stack([oracle.histogram(ids[r], w.E) for r in range(w.R)]).astype(np.int32)
    hist_all[1, 3] += 1                                # rank 1's row no longer matches its ids
    out = mep.RankPlanBuffers.allocate(w.R, w.E, w.S, w.K, dev())
    mep.mep_plan_rank(torch.from_numpy(ids[1].copy()).to(dev()), torch.from_numpy(hist_all).to(dev()),
                      w.R, w.E, w.S, w.K, 1, out)
    assert mep.mep_get_error() & mep.DERR_HIST
    mep.mep_plan_rank(torch.from_numpy(ids[0].copy()).to(dev()), torch.from_numpy(hist_all).to(dev()),
                      w.R, w.E, w.S, w.K, 0, out)
    assert mep.mep_get_error() == 0                    # rank 0's own row still matches
