"""Pins for the oracle's bf16 rounding, dispatch, int8 quantisation and combine.

Checked against a library routine (torch's float->bf16 conversion), exact results
with known closed forms, and the exact sum (in float64) within the error bound of a
binary32 accumulation followed by one bf16 rounding.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_float_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    specials = np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e38, 3.4e38,
                         np.inf, -np.inf, 1e-40, -1e-41, 1.1754944e-38, 65504.0, 0.1], np.float32)
    # exact ties between two bf16 values: low 16 bits == 0x8000
    ties = (rng.integers(0, 2**15, 64).astype(np.uint32) << 17 | 0x8000 |
            (rng.integers(0, 2, 64).astype(np.uint32) << 16)).view(np.float32)
    vals = np.concatenate([specials, ties, rng.standard_normal(2000).astype(np.float32) * 100,
                           rng.standard_normal(200).astype(np.float32) * 1e-39])
    vals = vals[np.isfinite(vals) | np.isinf(vals)]
    ours = oracle.float_to_bf16(vals)
    ref = _bits(torch.from_numpy(vals).to(torch.bfloat16))
    assert np.array_equal(ours, ref)
    nan = oracle.float_to_bf16(np.array([np.nan], np.float32))
    assert np.isnan(oracle.bf16_to_float(nan)).all()


def test_dispatch_copies_rows_to_their_positions():
    rng = np.random.default_rng(1)
    T, K, H = 7, 3, 40
    x = rng.integers(0, 2**16, (T, H)).astype(np.uint16)
    pos = rng.permutation(T * K + 5)[: T * K].astype(np.int32)
    pos[[2, 9]] = -1
    recv = oracle.dispatch(x, pos, K, T * K + 5)
    for n in range(T * K):
        if pos[n] >= 0:
            assert np.array_equal(recv[pos[n]], x[n // K])
    untouched = np.setdiff1d(np.arange(T * K + 5), pos[pos >= 0])
    assert not recv[untouched].any()
    with pytest.raises(oracle.OracleError):
        oracle.dispatch(x, np.full(T * K, T * K + 5, np.int32), K, T * K + 5)


def test_quant_half_even_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "quant_half_even.json")))
    xb = _bits(torch.tensor(g["x"], dtype=torch.bfloat16))
    assert np.array_equal(oracle.bf16_to_float(xb), np.array(g["x"], np.float32))
    q, s = oracle.quantize_row(xb)
    assert s == g["expected_scale"]
    assert q.tolist() == g["expected_q"]


def test_quant_properties():
    rng = np.random.default_rng(2)
    for trial in range(50):
        H = int(rng.integers(1, 300))
        scale_in = float(10.0 ** rng.uniform(-6, 4))
        xf = (rng.standard_normal(H) * scale_in).astype(np.float32)
        xb = _bits(torch.from_numpy(xf).to(torch.bfloat16))
        x = oracle.bf16_to_float(xb).astype(np.float64)
        q, s = oracle.quantize_row(xb)
        amax = np.abs(x).max()
        assert s == np.float32(np.float32(amax) / np.float32(127.0))
        assert q.min() >= -127 and q.max() <= 127
        j = int(np.argmax(np.abs(x)))
        assert abs(int(q[j])) == 127 and np.sign(q[j]) == np.sign(x[j])
        err = np.abs(q.astype(np.float64) * s - x)
        assert np.all(err <= 0.5 * s * (1 + 1e-5) + 1e-30)
    q, s = oracle.quantize_row(np.zeros(16, np.uint16))
    assert s == 0.0 and not q.any()


def test_dispatch_int8_all_copies_identical():
    rng = np.random.default_rng(3)
    T, K, H = 5, 4, 64
    x = _bits(torch.randn(T, H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16))
    pos = rng.permutation(T * K).astype(np.int32)
    q, sc = oracle.dispatch_int8(x, pos, K, T * K)
    for g in range(T):
        q0, s0 = oracle.quantize_row(x[g])
        for k in range(K):
            assert np.array_equal(q[pos[g * K + k]], q0) and sc[pos[g * K + k]] == s0


def test_dequantize_is_rounded_product():
    rng = np.random.default_rng(4)
    q = rng.integers(-127, 128, (6, 33)).astype(np.int8)
    s = rng.random(6).astype(np.float32)
    y = oracle.dequantize(q, s)
    ref = _bits((torch.from_numpy(q.astype(np.float32)) * torch.from_numpy(s)[:, None]).to(torch.bfloat16))
    assert np.array_equal(y, ref)


def test_combine_k1_is_one_rounded_product():
    rng = np.random.default_rng(5)
    T, H = 9, 50
    y = _bits(torch.randn(T, H, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16))
    g = rng.random(T).astype(np.float32)
    pos = rng.permutation(T).astype(np.int32)
    out = oracle.combine(y, pos, g, 1)
    ref = _bits((torch.from_numpy(g)[:, None] *
                 torch.from_numpy(oracle.bf16_to_float(y[pos]))).to(torch.bfloat16))
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("K", [1, 2, 4, 8, 16])
def test_combine_equal_power_of_two_gates_is_exact(K):
    """Identity expert, gates 1/K with K a power of two: every partial sum j*x/K is
    exact in binary32, so the output is x itself."""
    T, H = 6, 70
    x = _bits(torch.randn(T, H, generator=torch.Generator().manual_seed(K)).to(torch.bfloat16))
    pos = np.arange(T * K, dtype=np.int32)
    y = oracle.dispatch(x, pos, K, T * K)
    out = oracle.combine(y, pos, np.full(T * K, 1.0 / K, np.float32), K)
    assert np.array_equal(out, x)


def test_combine_softmax_gates_identity_expert_returns_x():
    """Gates summing to 1 (within fp32 rounding) on copies of x: the fp32 sum is
    x*(1+d) with |d| < 2^-9, which rounds back to x in bf16."""
    rng = np.random.default_rng(6)
    T, K, H = 20, 8, 64
    x = _bits(torch.randn(T, H, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16))
    z = rng.standard_normal((T, K))
    g = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    pos = rng.permutation(T * K).astype(np.int32)
    y = oracle.dispatch(x, pos, K, T * K)
    out = oracle.combine(y, pos, g, K)
    assert np.array_equal(out, x)


def test_combine_random_rows_within_error_bound():
    """Arbitrary expert rows and dropped slots: the output is the exact (float64) sum
    up to the binary32 accumulation error plus one bf16 rounding."""
    rng = np.random.default_rng(7)
    T, K, H, rows = 30, 6, 48, 200
    y = _bits(torch.randn(rows, H, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16))
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.2] = -1
    g = rng.random(T * K).astype(np.float32)
    out = oracle.bf16_to_float(oracle.combine(y, pos, g, K)).astype(np.float64)
    yf = oracle.bf16_to_float(y).astype(np.float64)
    for t in range(T):
        exact = np.zeros(H)
        mag = np.zeros(H)
        for k in range(K):
            p = pos[t * K + k]
            if p >= 0:
                exact += float(g[t * K + k]) * yf[p]
                mag += abs(float(g[t * K + k]) * yf[p])
        bound = 2.0 ** -8 * np.abs(exact) + (K + 1) * 2.0 ** -24 * mag * (1 + 2.0 ** -8) + 1e-38
        assert np.all(np.abs(out[t] - exact) <= bound)
        if np.all(pos[t * K:(t + 1) * K] < 0):
            assert not out[t].any()


def test_route_tokens_matches_whole_pipeline():
    rng = np.random.default_rng(8)
    T, K, H = 10, 4, 32
    x = _bits(torch.randn(T, H, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16))
    pos = rng.permutation(T * K).astype(np.int32)
    pos[[1, 5, 6]] = -1
    g = rng.random(T * K).astype(np.float32)
    for quant in (0, 1):
        if quant:
            q, sc = oracle.dispatch_int8(x, pos, K, T * K)
            y = oracle.dequantize(q, sc)
        else:
            y = oracle.dispatch(x, pos, K, T * K)
        full = oracle.combine(y, pos, g, K)
        one = oracle.route_tokens(x, (pos >= 0).reshape(T, K), g.reshape(T, K), K, quant)
        assert np.array_equal(full, one)


def test_combine_int8_identity_rows_return_the_dequantised_row():
    """int8 round trip with gates summing to 1: every token's K rows are the same codes
    and scale, so the combine gives back bf16(q*scale) of its row (as values)."""
    rng = np.random.default_rng(9)
    T, K, H = 12, 8, 96
    x = _bits((torch.randn(T, H, generator=torch.Generator().manual_seed(9)) * 7).to(torch.bfloat16))
    z = rng.standard_normal((T, K))
    g = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    pos = rng.permutation(T * K).astype(np.int32)
    q, sc = oracle.dispatch_int8(x, pos, K, T * K)
    out = oracle.combine_int8(q, sc, pos, g, K)
    for t in range(T):
        q0, s0 = oracle.quantize_row(x[t])
        row = oracle.bf16_to_float(oracle.dequantize(q0[None, :], np.array([s0], np.float32))[0])
        assert np.array_equal(oracle.bf16_to_float(out[t]), row)


def test_combine_int8_k1_is_rounded_product_of_rounded_dequant():
    rng = np.random.default_rng(10)
    T, H = 7, 40
    q = rng.integers(-127, 128, (T, H)).astype(np.int8)
    sc = rng.random(T).astype(np.float32)
    g = rng.random(T).astype(np.float32)
    pos = np.arange(T, dtype=np.int32)
    out = oracle.combine_int8(q, sc, pos, g, 1)
    y = (torch.from_numpy(q.astype(np.float32)) * torch.from_numpy(sc)[:, None]).to(torch.bfloat16).float()
    ref = _bits((torch.from_numpy(g)[:, None] * y).to(torch.bfloat16))
    assert np.array_equal(out, ref)
