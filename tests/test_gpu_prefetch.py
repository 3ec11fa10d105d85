"""GPU parity of the replica weight prefetch (slot plan and copy) and the replica
gradient reduce against the oracle, plus full-size properties on the r8 workload with
MoonEP's benchmark expert width H' = 2048."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu


def _gpu_prefetch_plan(pb, R, E, B):
    cap = pb.rep_key.shape[1]
    se = torch.empty((R, max(B, 1)), dtype=torch.int32, device=dev())[:, :B].contiguous()
    rw = torch.empty((R, cap), dtype=torch.int32, device=dev())
    mep.mep_prefetch_plan(pb, R, E, B, se, rw)
    return se, rw


@pytest.mark.parametrize("name,B", [("tiny", 4), ("r8", 8), ("r8", 3), ("skew", 8), ("skew", 1),
                                    ("int8", 8), ("r8", 0)])
def test_prefetch_plan_parity(name, B):
    w = synth.get(name)
    ids, _ = synth.router(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    se, rw = _gpu_prefetch_plan(pb, w.R, w.E, B)
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    ose, orw = oracle.prefetch_plan(p.rep_count, p.rep_key, w.R, w.E, B)
    assert np.array_equal(se.cpu().numpy(), ose)
    assert np.array_equal(rw.cpu().numpy(), orw)
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("D", [64, 1000, 33, 7])
def test_prefetch_weights_and_grad_reduce_small(D):
    rng = np.random.default_rng(D)
    E, R, B = 12, 4, 5
    se = np.full((R, B), -1, np.int32)
    for r in range(R):
        n = rng.integers(0, B + 1)
        se[r, :n] = rng.choice(E, size=n, replace=False)
    se[0, 0] = 3
    se[2, 0] = 3                                  # an expert prefetched by several ranks
    w_home = rng.integers(0, 2 ** 16, (E, D)).astype(np.uint16)
    w_slots0 = rng.integers(0, 2 ** 16, (R * B, D)).astype(np.uint16)
    ws = torch.from_numpy(w_slots0.view(np.int16)).to(dev()).view(torch.bfloat16)
    mep.mep_prefetch_weights(torch.from_numpy(w_home.view(np.int16)).to(dev()).view(torch.bfloat16),
                             torch.from_numpy(se).to(dev()), R, B, ws)
    assert np.array_equal(bits(ws), oracle.prefetch_weights(w_home, se, R, B, w_slots0))
    gh = (rng.standard_normal((E, D)) * 10.0 ** rng.uniform(-3, 3, (E, 1))).astype(np.float32)
    gs = (rng.standard_normal((R * B, D)) * 10.0 ** rng.uniform(-3, 3, (R * B, 1))).astype(np.float32)
    gh_d, gs_d = torch.from_numpy(gh).to(dev()), torch.from_numpy(gs).to(dev())
    mep.mep_grad_reduce(gh_d, gs_d, torch.from_numpy(se).to(dev()), R, B)
    oh, os_ = oracle.grad_reduce(gh, gs, se, R, B)
    assert np.array_equal(gh_d.cpu().numpy().view(np.uint32), oh.view(np.uint32))
    assert np.array_equal(gs_d.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert mep.mep_get_error() == 0


def test_prefetch_and_grad_reduce_full_r8():
    """R8 E64 S4096, B = E/R = 8, H' = 2048 (14.7M elements per expert): every used
    slot holds its expert's weights; every expert's gradient equals its home gradient
    plus its slots in ascending order (fp32 adds by torch in the same order), and the
    slots are cleared."""
    w = synth.get("r8")
    Hf = 2048
    D = w.H * Hf
    B = w.E // w.R
    ids, _ = synth.router(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    se, rw = _gpu_prefetch_plan(pb, w.R, w.E, B)
    g = torch.Generator(device=dev()).manual_seed(0)
    w_home = torch.randn((w.E, D), generator=g, device=dev()).to(torch.bfloat16)
    w_slots = torch.zeros((w.R * B, D), dtype=torch.bfloat16, device=dev())
    mep.mep_prefetch_weights(w_home, se, w.R, B, w_slots)
    flat = se.view(-1).long()
    used = torch.nonzero(flat >= 0).view(-1)
    assert used.numel() == min(pb.stats_dict()["prefetched"], w.R * B)
    for s in used.tolist():
        assert torch.equal(w_slots[s].view(torch.int16), w_home[flat[s]].view(torch.int16))
    del w_home, w_slots
    grad_home = torch.randn((w.E, D), generator=g, device=dev())
    grad_slots = torch.randn((w.R * B, D), generator=g, device=dev())
    want = grad_home.clone()
    for s in used.tolist():                      # ascending slot order, one fp32 add each
        want[flat[s]] = want[flat[s]] + grad_slots[s]
    keep_unused = grad_slots[flat < 0].clone()
    mep.mep_grad_reduce(grad_home, grad_slots, se, w.R, B)
    assert torch.equal(grad_home.view(torch.int32), want.view(torch.int32))
    assert not grad_slots[used].any()
    assert torch.equal(grad_slots[flat < 0], keep_unused)
    assert mep.mep_get_error() == 0
