"""GPU parity of the int8 dispatch with per-expert smoothing scales against the oracle
(codes and scales bit for bit; K in {2, 4, 8} takes the fused kernel, the others the
per-slot one), and the special case of all-ones scales against the plain per-token int8
dispatch on the full int8 workload."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("H", [8, 64, 4096, 7168, 12288, 20000, 7])
def test_smooth_dispatch_matches_oracle(K, H):
    rng = np.random.default_rng(K * 7 + H)
    T, E = 23, 10
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(H)) * 4).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    rows = T * K + 2
    pos = rng.permutation(rows)[: T * K].astype(np.int32)
    pos[rng.random(T * K) < 0.15] = -1
    sm = (10.0 ** rng.uniform(-2, 2, (E, H))).astype(np.float32)
    q = torch.zeros((rows, H), dtype=torch.int8, device=dev())
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


def test_smooth_dispatch_full_int8_workload():
    w = synth.get("int8")
    ids, _ = synth.router(w)
    x = synth.hidden(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    x_d = x.to(dev())
    ids_d = torch.from_numpy(ids).to(dev()).view(-1)
    q = torch.empty((w.N, w.H), dtype=torch.int8, device=dev())
    sc = torch.empty(w.N, dtype=torch.float32, device=dev())
    # all-ones scales: the plain per-token int8 dispatch, every row
    mep.mep_dispatch_int8_smooth(x_d, ids_d, pb.pos, w.K, torch.ones((w.E, w.H), device=dev()), q, sc)
    q0 = torch.empty_like(q)
    s0 = torch.empty_like(sc)
    mep.mep_dispatch(x_d, pb.pos, w.K, q0, s0, quant=1)
    assert torch.equal(q, q0) and torch.equal(sc.view(torch.int32), s0.view(torch.int32))
    # per-expert scales: sampled tokens, every slot, against the oracle
    rng = np.random.default_rng(21)
    sm = (10.0 ** rng.uniform(-1, 1, (w.E, w.H))).astype(np.float32)
    mep.mep_dispatch_int8_smooth(x_d, ids_d, pb.pos, w.K, torch.from_numpy(sm).to(dev()), q, sc)
    pos = pb.pos.cpu().numpy()
    for t in np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, 60)])):
        sl = slice(t * w.K, (t + 1) * w.K)
        q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x[t:t + 1]), ids[t][None, :],
                                                   np.arange(w.K, dtype=np.int32), w.K, sm, w.K)
        rows = torch.from_numpy(pos[sl].astype(np.int64)).to(dev())
        assert np.array_equal(q[rows].cpu().numpy(), q_ref)
        assert np.array_equal(sc[rows].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("amax", [381.0, 88.9, 1.0e-3, 5.0e30, 1.0e-36])
def test_quantiser_at_and_next_to_half_integer_quotients(amax):
    """Codes of values whose quotient by the scale sits on or within a few ulps of a
    half-integer, where a quotient taken through the reciprocal could round the other
    way: with x = 1, the smoothing scales are the quantised values themselves. Column 0
    holds amax (so scale = fl(amax / 127)); the others are fl(scale * (k + 0.5)) and its
    neighbours 1 and 2 ulps away, for every k from -127 to 126."""
    sc32 = np.float32(np.float32(amax) / np.float32(127.0))
    vals = [np.float32(amax)]
    for k in range(-127, 127):
        c = np.float32(sc32 * np.float32(k + 0.5))
        for j in (-2, -1, 0, 1, 2):
            v = c
            for _ in range(abs(j)):
                v = np.nextafter(v, np.float32(np.inf if j > 0 else -np.inf), dtype=np.float32)
            if abs(v) <= np.float32(amax):
                vals.append(v)
    H = (len(vals) + 7) // 8 * 8
    sm = np.zeros((1, H), np.float32)
    sm[0, :len(vals)] = vals
    x = torch.ones((1, H), dtype=torch.bfloat16)
    ids = np.zeros((1, 1), np.int32)
    pos = np.zeros(1, np.int32)
    q = torch.zeros((1, H), dtype=torch.int8, device=dev())
    s = torch.zeros(1, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), 1, torch.from_numpy(sm).to(dev()), q, s)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, 1, sm, 1)
    assert s_ref[0] == sc32
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0
