"""Pins for the oracle's combine + residual add + RMSNorm and its binary64 -> bf16
rounding: torch's rms_norm in float64 (a library routine), closed forms, and rounding
cases where a detour through binary32 would round twice."""
import numpy as np
import torch

import oracle


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_double_to_bf16_single_rounding():
    rng = np.random.default_rng(0)
    f = (rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000)).astype(np.float32)
    # values exact in binary32: one rounding either way, so torch's conversion agrees
    assert np.array_equal(oracle.double_to_bf16(f.astype(np.float64)),
                          _bits(torch.from_numpy(f).to(torch.bfloat16)))
    # a tie in binary32 that is not a tie in binary64 must round away from it
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80          # exact tie -> even
    assert oracle.double_to_bf16(-(1.0 + 3 * 2.0 ** -8)) == 0xBF82    # tie -> even (up)
    assert oracle.double_to_bf16(1.5 * 2.0 ** -133) == 0x0002         # subnormal tie -> even
    assert oracle.double_to_bf16(0.0) == 0 and oracle.double_to_bf16(-0.0) == 0x8000


def _case(T, K, H, rows, seed):
    rng = np.random.default_rng(seed)
    g = torch.Generator().manual_seed(seed)
    y = _bits(torch.randn(rows, H, generator=g).to(torch.bfloat16))
    res = _bits((torch.randn(T, H, generator=g) * 0.5).to(torch.bfloat16))
    gam = _bits((1.0 + 0.1 * torch.randn(H, generator=g)).to(torch.bfloat16))
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.15] = -1
    gates = rng.random(T * K).astype(np.float32)
    return y, res, gam, pos, gates


def test_rmsnorm_matches_torch_float64():
    T, K, H, rows, eps = 17, 4, 96, 80, 1e-6
    y, res, gam, pos, gates = _case(T, K, H, rows, 1)
    x_out, y_out, y_exact, rstd = oracle.combine_add_rmsnorm(y, pos, gates, K, res, gam, eps)
    c = oracle.combine(y, pos, gates, K)
    x = torch.from_numpy(oracle.bf16_to_float(c).astype(np.float64) +
                         oracle.bf16_to_float(res).astype(np.float64))
    w = torch.from_numpy(oracle.bf16_to_float(gam).astype(np.float64))
    ref = torch.nn.functional.rms_norm(x, (H,), weight=w, eps=eps).numpy()
    assert np.allclose(y_exact, ref, rtol=1e-12, atol=0)
    assert np.array_equal(y_out, oracle.double_to_bf16(ref))
    # x_out: the exact sum rounded once; where the sum is exact in binary32 torch agrees
    xf = x.numpy().astype(np.float32)
    exact32 = xf.astype(np.float64) == x.numpy()
    tb = _bits(torch.from_numpy(xf).to(torch.bfloat16))
    assert np.array_equal(x_out[exact32], tb[exact32])


def test_rmsnorm_constant_rows_closed_form():
    """Every column of a token equal to a, gamma = 1: rstd = 1/sqrt(a^2 + eps), y = a*rstd."""
    T, K, H, eps = 5, 1, 64, 1e-5
    vals = np.array([0.5, -3.0, 1e-3, 0.0, 40.0])
    y = np.repeat(oracle.float_to_bf16(vals.astype(np.float32))[:, None], H, axis=1)
    res = np.zeros((T, H), np.uint16)
    gam = np.full(H, 0x3F80, np.uint16)
    pos = np.arange(T, dtype=np.int32)
    gates = np.ones(T, np.float32)
    x_out, y_out, y_exact, rstd = oracle.combine_add_rmsnorm(y, pos, gates, K, res, gam, eps)
    a = oracle.bf16_to_float(y[:, 0]).astype(np.float64)
    assert np.allclose(rstd, 1.0 / np.sqrt(a * a + eps), rtol=1e-15)
    assert np.allclose(y_exact, (a / np.sqrt(a * a + eps))[:, None], rtol=1e-15)
    assert np.array_equal(x_out, y)


def test_rmsnorm_dropped_token_is_the_residual():
    """A token with every slot dropped combines to zero: x is its residual row."""
    T, K, H, rows, eps = 3, 2, 32, 4, 1e-6
    y, res, gam, pos, gates = _case(T, K, H, rows, 2)
    pos[:] = -1
    x_out, _, _, _ = oracle.combine_add_rmsnorm(y, pos, gates, K, res, gam, eps)
    assert np.array_equal(oracle.bf16_to_float(x_out), oracle.bf16_to_float(res))
