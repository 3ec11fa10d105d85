"""Pins for the oracle's smooth-quantised int8 dispatch: all-ones scales reduce to the
plain per-token int8 dispatch; power-of-two scales commute with the quantisation
exactly; per-slot quantisation bounds."""
import numpy as np
import torch

import oracle


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _case(seed, T=9, K=4, H=64, E=6):
    rng = np.random.default_rng(seed)
    x = _bits((torch.randn(T, H, generator=torch.Generator().manual_seed(seed)) * 3).to(torch.bfloat16))
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    pos = rng.permutation(T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.2] = -1
    return rng, x, ids, pos, E


def test_smooth_ones_is_the_plain_int8_dispatch():
    rng, x, ids, pos, E = _case(1)
    T, H = x.shape
    K = ids.shape[1]
    q, sc = oracle.dispatch_int8_smooth(x, ids, pos, K, np.ones((E, H), np.float32), T * K)
    q0, sc0 = oracle.dispatch_int8(x, pos, K, T * K)
    assert np.array_equal(q, q0) and np.array_equal(sc.view(np.uint32), sc0.view(np.uint32))


def test_power_of_two_scales_commute_with_quantisation():
    """xs = x * 2^k exactly; amax and scale scale by 2^k; xs/scale = x/scale': the codes
    are the plain ones and the scale is multiplied by 2^k."""
    rng, x, ids, pos, E = _case(2)
    T, H = x.shape
    K = ids.shape[1]
    k = rng.integers(-6, 7, E)
    sm = np.repeat((2.0 ** k).astype(np.float32)[:, None], H, axis=1)
    q, sc = oracle.dispatch_int8_smooth(x, ids, pos, K, sm, T * K)
    q0, sc0 = oracle.dispatch_int8(x, pos, K, T * K)
    kept = pos >= 0
    rows = pos[kept]
    assert np.array_equal(q[rows], q0[rows])
    assert np.array_equal(sc[rows], (sc0[rows] * (2.0 ** k[ids.ravel()[kept]])).astype(np.float32))


def test_per_slot_bounds():
    rng, x, ids, pos, E = _case(3, T=12, K=3, H=100, E=5)
    T, H = x.shape
    K = ids.shape[1]
    sm = (10.0 ** rng.uniform(-2, 2, (E, H))).astype(np.float32)
    q, sc = oracle.dispatch_int8_smooth(x, ids, pos, K, sm, T * K)
    xf = oracle.bf16_to_float(x).astype(np.float32)
    for n in np.flatnonzero(pos >= 0):
        xs = (xf[n // K] * sm[ids.ravel()[n]]).astype(np.float32).astype(np.float64)
        row, s = q[pos[n]].astype(np.float64), float(sc[pos[n]])
        assert s == np.float32(np.float32(np.abs(xs).max()) / np.float32(127))
        assert np.all(np.abs(row * s - xs) <= 0.5 * s * (1 + 1e-5))
        assert abs(row[np.argmax(np.abs(xs))]) == 127
