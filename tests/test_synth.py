"""The seeded input generator: shapes, determinism and the properties the pages
require of router outputs and mapping inputs."""
import numpy as np
import torch

import synth


def test_router_outputs_are_valid_and_deterministic():
    for name in ["tiny", "map"]:
        w = synth.get(name)
        ids, gates = synth.router(w)
        ids2, gates2 = synth.router(w, threads=1)
        assert np.array_equal(ids, ids2) and np.array_equal(gates, gates2)
        assert ids.shape == (w.T, w.K) and ids.dtype == np.int32
        assert ids.min() >= 0 and ids.max() < w.E
        assert all(len(set(r)) == w.K for r in ids.tolist())          # no repeats in a token
        assert np.all(np.diff(gates, axis=1) <= 0)                       # descending
        assert np.allclose(gates.sum(1), 1.0, atol=1e-5)


def test_skew_forces_expert0_and_zipf_is_skewed():
    w = synth.scaled(synth.get("skew"), S=32)
    ids, gates = synth.router(w)
    assert np.all((ids == 0).sum(1) == 1)
    h = np.bincount(ids.ravel(), minlength=w.E)
    assert h[0] == w.T and h.max() == w.T


def test_hidden_rows_and_outliers():
    w = synth.scaled(synth.get("int8"), S=64, H=256)
    x = synth.hidden(w)
    assert x.dtype == torch.bfloat16 and x.shape == (w.T, w.H)
    assert torch.equal(x, synth.hidden(w, threads=3))
    amax = x.float().abs().amax(1)
    n_out = int(round(w.outlier_frac * w.T))
    assert (amax > 30).sum().item() >= n_out // 2


def test_mapping_table_is_well_formed():
    w = synth.get("map")
    table, thr, active = synth.mapping_inputs(w)
    assert table.shape == (w.E, w.F)
    assert set(table[:, 0].tolist()) <= {1, 2} and (table[:, 0] == 2).sum() == w.n_hot
    ids = np.concatenate([table[e, 1:1 + table[e, 0]] for e in range(w.E)])
    assert sorted(ids.tolist()) == list(range(w.R * w.place_per_rank))
    assert np.bincount(ids // w.place_per_rank).tolist() == [w.place_per_rank] * w.R
    assert thr.shape == (w.K,) and np.all((thr >= 0) & (thr < 0.1))
    assert active.reshape(w.R, w.S)[:, : w.n_active].all() and not active.reshape(w.R, w.S)[:, w.n_active:].any()


def test_router_follows_the_zipf_bias():
    """Experts with a larger Zipf bias receive more slots: the per-expert counts rank like
    the bias (Spearman correlation), the first expert leads when there is no
    permutation, and a permuted workload does not keep the identity order."""
    for name, S in [("tiny", 128), ("r8", 256), ("int8", 256)]:
        w = synth.scaled(synth.get(name), S=S)
        ids, _ = synth.router(w)
        h = np.bincount(ids.ravel(), minlength=w.E).astype(np.float64)
        bias, rank = synth.zipf_bias(w)
        rh = np.argsort(np.argsort(-h))
        rb = np.argsort(np.argsort(-bias))
        rho = np.corrcoef(rh, rb)[0, 1]
        assert rho > 0.8, (name, rho)
        if not w.permute:
            assert h.argmax() == 0
        else:
            assert not np.array_equal(rank, np.arange(w.E))


def test_hidden_rows_are_standard_normal_in_bf16():
    w = synth.scaled(synth.get("r8"), S=8, H=1024)
    x = synth.hidden(w).float()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    # every value is a bf16 number (rounded once from the fp32 draw)
    assert torch.equal(x.to(torch.bfloat16).float(), x)
