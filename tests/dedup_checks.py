"""Properties every deduplicated dispatch encoding of a plan must have (shared by the
oracle pins and the GPU parity tests)."""
import numpy as np


def _rank_of(rows, rank_off):
    return np.searchsorted(rank_off, rows, side="right") - 1


def check_dedup(pos, K, rank_off, d):
    """Every property a deduplicated encoding of this plan must have."""
    N = pos.size
    T = N // K
    R = rank_off.size - 1
    kept = np.nonzero(pos >= 0)[0]
    g = kept // K
    r = _rank_of(pos[kept], rank_off)
    pairs = np.unique(np.stack([r, g], 1), axis=0)           # sorted by rank, then token
    U = int(d.drank_off[R])
    assert U == pairs.shape[0]
    # rows of rank r: its tokens in ascending order, each once
    assert np.array_equal(d.dtok[:U], pairs[:, 1])
    assert np.array_equal(d.drank_off, np.searchsorted(pairs[:, 0], np.arange(R + 1), side="left"))
    assert (d.dtok[U:] == -1).all()
    # every kept slot points at the row of its own (token, rank) pair
    assert (d.dpos[pos < 0] == -1).all() and (d.dsend[pos < 0] == -1).all()
    assert np.array_equal(d.dtok[d.dpos[kept]], g)
    assert np.array_equal(_rank_of(d.dpos[kept], d.drank_off), r)
    # the send list names each pair once, at its first slot
    sent = np.nonzero(d.dsend >= 0)[0]
    assert np.array_equal(np.sort(d.dsend[sent]), np.arange(U))
    for n in sent:
        gg = n // K
        same = [m for m in range(gg * K, n) if pos[m] >= 0 and _rank_of(pos[m], rank_off) == _rank_of(pos[n], rank_off)]
        assert not same and d.dpos[n] == d.dsend[n]
    # gidx inverts the plan rows
    assert np.array_equal(d.gidx[pos[kept]], d.dpos[kept])
    assert (d.gidx[rank_off[R]:] == -1).all()
    # bounds: a rank receives each token at most once and never more rows than slots
    per_rank = np.diff(d.drank_off)
    assert (per_rank <= T).all() and (per_rank <= np.diff(rank_off)).all()
    assert np.unique(g).size <= U <= kept.size
