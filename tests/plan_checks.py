"""Properties every placement plan must have, whatever computed it."""
import numpy as np


def check_balanced_plan(ids, R, E, S, K, pos, rep_count, rep_key, rep_cu, redundant):
    """The MoonEP invariants: every rank gets exactly S*K rows; each slot lands in a
    replica of its own expert; a replica's rows are contiguous and in (src, t, k) order;
    at most R-1 redundant replicas."""
    ids = np.asarray(ids, np.int64).ravel()
    N, SK = R * S * K, S * K
    pos = np.asarray(pos, np.int64)
    assert pos.shape == (N,)
    # a permutation of [0, N): every rank's chunk is exactly full
    assert np.array_equal(np.sort(pos), np.arange(N))
    assert np.all(np.bincount(pos // SK, minlength=R) == SK)
    row_key = np.empty(N, np.int64)
    row_key[pos] = ids
    row_slot = np.empty(N, np.int64)
    row_slot[pos] = np.arange(N)
    for r in range(R):
        c = int(rep_count[r])
        cu = np.asarray(rep_cu[r][: c + 1], np.int64)
        keys = np.asarray(rep_key[r][:c], np.int64)
        assert cu[0] == 0 and cu[-1] == SK
        assert np.all(np.diff(cu) > 0)
        assert np.all(np.diff(keys) > 0)          # ascending experts, each once
        for j in range(c):
            lo, hi = r * SK + cu[j], r * SK + cu[j + 1]
            assert np.all(row_key[lo:hi] == keys[j])
            assert np.all(np.diff(row_slot[lo:hi]) > 0)   # (src, t, k) order
    assert 0 <= redundant <= R - 1
