"""GPU parity of the combine fused with residual add and RMSNorm.

x_out is compared bit for bit (the sum rounded once). y_out and rstd come from an fp32
sum of H squares whose order is the kernel's; they are compared with the oracle's
binary64 values within the bound that order allows:
  rstd: relative ((H+3)/2 + 2) * 2^-24      (fp32 sum of H squares, division, rsqrt)
  y:    0.5 bf16 ulp + the same relative error plus three more fp32 roundings,
        which is always within 1 bf16 ulp.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _bf16_ulp(v):
    v = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(v)) - 7)


def _check(got_x, got_y, got_r, x_ref, y_exact, rstd_ref, H):
    assert np.array_equal(got_x, x_ref)
    rel = ((H + 3) / 2 + 2) * U
    assert np.all(np.abs(got_r.astype(np.float64) - rstd_ref) <= rel * rstd_ref)
    yg = oracle.bf16_to_float(got_y).astype(np.float64)
    big = np.maximum(np.abs(y_exact), np.abs(yg))
    bound = 0.5 * _bf16_ulp(big) + (rel + 4 * U) * np.abs(y_exact) + 2.0 ** -133
    assert np.all(np.abs(yg - y_exact) <= bound)
    assert np.all(np.abs(yg - y_exact) <= _bf16_ulp(big))


@pytest.mark.parametrize("K", [1, 2, 3, 4, 6, 8])
@pytest.mark.parametrize("H", [8, 96, 4096, 7168, 7, 130])
def test_combine_add_rmsnorm_small(K, H):
    rng = np.random.default_rng(K * 100 + H)
    T, rows, eps = 37, 200, 1e-6
    g = torch.Generator().manual_seed(K + H)
    y = (torch.randn(rows, H, generator=g) * 3).to(torch.bfloat16)
    res = (torch.randn(T, H, generator=g)).to(torch.bfloat16)
    gam = (1.0 + 0.2 * torch.randn(H, generator=g)).to(torch.bfloat16)
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[rng.random(T * K) < 0.15] = -1
    pos[:K] = -1                                   # token 0: residual only
    gates = rng.random(T * K).astype(np.float32)
    x_out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    y_out = torch.empty_like(x_out)
    rstd = torch.empty(T, dtype=torch.float32, device=dev())
    mep.mep_combine_add_rmsnorm(y.to(dev()), torch.from_numpy(pos).to(dev()),
                                torch.from_numpy(gates).to(dev()), K, res.to(dev()), gam.to(dev()),
                                eps, x_out, y_out, rstd)
    xr, _, ye, rr = oracle.combine_add_rmsnorm(bits(y), pos, gates, K, bits(res), bits(gam), eps)
    _check(bits(x_out), bits(y_out), rstd.cpu().numpy(), xr, ye, rr, H)
    assert mep.mep_get_error() == 0


def test_combine_add_rmsnorm_full_r8():
    """Full-size r8 workload, identity expert: every row's x_out equals bf16(x + residual)
    (the combine gives x back exactly), sampled tokens match the oracle."""
    w = synth.get("r8")
    ids, gates = synth.router(w)
    x = synth.hidden(w)
    res = synth.expert_outputs(synth.scaled(w, S=w.S), w.T)
    gam = (1.0 + 0.1 * torch.randn(w.H, generator=torch.Generator().manual_seed(5))).to(torch.bfloat16)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    x_d, res_d = x.to(dev()), res.to(dev())
    recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev())
    mep.mep_dispatch(x_d, pb.pos, w.K, recv)
    x_out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
    y_out = torch.empty_like(x_out)
    rstd = torch.empty(w.T, dtype=torch.float32, device=dev())
    mep.mep_combine_add_rmsnorm(recv, pb.pos, torch.from_numpy(gates).to(dev()), w.K, res_d,
                                gam.to(dev()), 1e-6, x_out, y_out, rstd)
    torch.cuda.synchronize()
    assert torch.equal(x_out.float(), (x_d.float() + res_d.float()).to(torch.bfloat16).float())
    toks = np.unique(np.concatenate([[0, w.T - 1], np.random.default_rng(3).integers(0, w.T, 40)]))
    for t in toks:
        posk = np.arange(w.K, dtype=np.int32)
        yk = oracle.dispatch(bits(x[t:t + 1]), posk, w.K, w.K)
        xr, _, ye, rr = oracle.combine_add_rmsnorm(yk, posk, gates[t], w.K, bits(res[t:t + 1]),
                                                    bits(gam), 1e-6)
        ti = int(t)
        _check(bits(x_out[ti:ti + 1]), bits(y_out[ti:ti + 1]), rstd[ti:ti + 1].cpu().numpy(),
               xr, ye, rr, w.H)
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("H", [49152, 49144, 49151])
def test_combine_add_rmsnorm_largest_rows(H):
    """The widest rows the fused kernel takes (H = MEP_RMSNORM_MAX_H = 49,152 floats of
    shared memory), ragged widths just below it (vector and element paths); one past it
    is refused."""
    rng = np.random.default_rng(H)
    T, K, rows, eps = 5, 4, 12, 1e-6
    g = torch.Generator().manual_seed(H)
    y = torch.randn(rows, H, generator=g).to(torch.bfloat16)
    res = torch.randn(T, H, generator=g).to(torch.bfloat16)
    gam = (1.0 + 0.2 * torch.randn(H, generator=g)).to(torch.bfloat16)
    pos = rng.integers(0, rows, T * K).astype(np.int32)
    pos[3] = -1
    gates = rng.random(T * K).astype(np.float32)
    x_out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    y_out = torch.empty_like(x_out)
    rstd = torch.empty(T, dtype=torch.float32, device=dev())
    mep.mep_combine_add_rmsnorm(y.to(dev()), torch.from_numpy(pos).to(dev()), torch.from_numpy(gates).to(dev()),
                                K, res.to(dev()), gam.to(dev()), eps, x_out, y_out, rstd)
    xr, _, ye, rr = oracle.combine_add_rmsnorm(bits(y), pos, gates, K, bits(res), bits(gam), eps)
    _check(bits(x_out), bits(y_out), rstd.cpu().numpy(), xr, ye, rr, H)
    assert mep.mep_get_error() == 0
    H1 = 49153
    with pytest.raises(mep.MepError) as e:
        mep.mep_combine_add_rmsnorm(torch.zeros((rows, H1), dtype=torch.bfloat16, device=dev()),
                                    torch.from_numpy(pos).to(dev()), torch.from_numpy(gates).to(dev()), K,
                                    torch.zeros((T, H1), dtype=torch.bfloat16, device=dev()),
                                    torch.zeros(H1, dtype=torch.bfloat16, device=dev()), eps,
                                    torch.empty((T, H1), dtype=torch.bfloat16, device=dev()),
                                    torch.empty((T, H1), dtype=torch.bfloat16, device=dev()), rstd)
    assert e.value.status == 3
