"""GPU parity of the int8 dispatch with per-expert smoothing scales against the oracle
(codes and scales bit for bit). H % 4 == 0 (up to 64 columns per thread, in groups of 4)
takes the fused kernel (all K slots of a token in one CTA, two passes, any K), other H or
alignments the scalar kernel. The full int8 workload is compared
whole, one rank partition at a time, and with all-ones scales against the plain
per-token int8 dispatch."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K", [1, 2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("H", [8, 12, 64, 4096, 4100, 7168, 12288, 16384, 16388, 20000, 7])
def test_smooth_dispatch_matches_oracle(K, H):
    rng = np.random.default_rng(K * 7 + H)
    T, E = 23, max(10, K + 3)
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


@pytest.mark.parametrize("K,H", [(2, 4096), (4, 7168), (8, 4096), (8, 12288), (8, 7168)])
def test_smooth_dispatch_many_tokens_per_cta(K, H):
    """More tokens than CTAs resident on the GPU, so every CTA walks many tokens;
    dropped slots and whole buffers."""
    rng = np.random.default_rng(K * 13 + H)
    T, E = 3001, 40
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(H + K)) * 3).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    rows = T * K + 5
    pos = rng.permutation(rows)[: T * K].astype(np.int32)
    pos[rng.random(T * K) < 0.1] = -1
    sm = (10.0 ** rng.uniform(-1.5, 1.5, (E, H))).astype(np.float32)
    q = torch.zeros((rows, H), dtype=torch.int8, device=dev())
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("x_off,q_off", [(4, 4), (4, 0), (0, 4), (1, 0), (0, 1)])
def test_smooth_dispatch_offset_buffers(x_off, q_off):
    """Token rows and receive rows that start off their usual alignment: an x 8 bytes and
    a receive buffer 4 bytes off 16 still take the kernel of 4-column groups; 2-byte or
    1-byte offsets take the scalar kernel. Same codes and scales either way."""
    rng = np.random.default_rng(100 * x_off + q_off)
    T, E, K, H = 37, 12, 8, 1028
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(x_off)) * 2).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    rows = T * K + 3
    pos = rng.permutation(rows)[: T * K].astype(np.int32)
    pos[rng.random(T * K) < 0.1] = -1
    sm = (10.0 ** rng.uniform(-1, 1, (E, H))).astype(np.float32)
    xb = torch.zeros(T * H + x_off, dtype=torch.bfloat16, device=dev())
    xv = xb[x_off:].view(T, H)
    xv.copy_(x.to(dev()))
    qb = torch.zeros(rows * H + q_off, dtype=torch.int8, device=dev())
    qv = qb[q_off:].view(rows, H)
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(xv, torch.from_numpy(ids).to(dev()).view(-1), torch.from_numpy(pos).to(dev()), K,
                                 torch.from_numpy(sm).to(dev()), qv, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(qv.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


def test_smooth_dispatch_bad_ids_and_rows_are_skipped_and_flagged():
    T, K, H, E = 64, 4, 4096, 8
    rng = np.random.default_rng(5)
    x = torch.randn((T, H), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    pos = np.arange(T * K, dtype=np.int32)
    ids[3, 1] = E + 2                                      # expert out of range: slot skipped
    sm = np.ones((E, H), np.float32)
    q = torch.full((T * K + 1, H), 55, dtype=torch.int8, device=dev())
    sc = torch.full((T * K + 1,), 7.0, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q[: T * K],
                                 sc[: T * K])
    assert mep.mep_get_error() & mep.DERR_KEY_RANGE
    assert bool((q[3 * K + 1] == 55).all()) and sc[3 * K + 1].item() == 7.0
    assert bool((q[T * K] == 55).all())                     # the guard row is untouched
    keep = np.ones(T * K, bool)
    keep[3 * K + 1] = False
    pos_ok = np.where(keep, pos, -1).astype(np.int32)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), np.where(ids < E, ids, 0), pos_ok, K, sm, T * K)
    got = q[: T * K].cpu().numpy()
    assert np.array_equal(got[keep], q_ref[keep])
    pos_bad = pos.copy()
    pos_bad[10] = T * K + 1                                # row out of range: slot skipped
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(np.where(ids < E, ids, 0)).to(dev()).view(-1),
                                 torch.from_numpy(pos_bad).to(dev()), K, torch.from_numpy(sm).to(dev()), q[: T * K],
                                 sc[: T * K])
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE


def test_smooth_dispatch_full_int8_workload():
    """The whole int8 workload: every code and scale against the oracle, one rank
    partition at a time; with all-ones scales, the plain per-token int8 dispatch."""
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
    del q0, s0
    # per-expert scales: every slot against the oracle
    rng = np.random.default_rng(21)
    sm = (10.0 ** rng.uniform(-1, 1, (w.E, w.H))).astype(np.float32)
    mep.mep_dispatch_int8_smooth(x_d, ids_d, pb.pos, w.K, torch.from_numpy(sm).to(dev()), q, sc)
    torch.cuda.synchronize()
    p = oracle.plan_balanced(ids, w.R, w.E, w.S, w.K)
    assert np.array_equal(pb.pos.cpu().numpy(), p.pos)
    xb = bits(x)
    SK = w.S * w.K

    def one(r):
        lo, hi = r * SK, (r + 1) * SK
        inside = (p.pos >= lo) & (p.pos < hi)
        toks = np.unique(np.flatnonzero(inside) // w.K)
        pos_r = np.where(inside, p.pos - lo, -1).astype(np.int32).reshape(-1, w.K)[toks]
        q_ref, s_ref = oracle.dispatch_int8_smooth(xb[toks], ids[toks], pos_r, w.K, sm, SK)
        assert np.array_equal(q[lo:hi].cpu().numpy(), q_ref), r
        assert np.array_equal(sc[lo:hi].cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), r
        return r
    with ThreadPoolExecutor(8) as ex:
        assert sorted(ex.map(one, range(w.R))) == list(range(w.R))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("K", [1, 2])
@pytest.mark.parametrize("amax", [381.0, 88.9, 1.0e-3, 5.0e30, 1.0e-36])
def test_quantiser_at_and_next_to_half_integer_quotients(amax, K):
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
    # K = 1: one slot; K = 2: the second slot on a second expert holding the values
    # reversed
    H = (len(vals) + 7) // 8 * 8
    sm = np.zeros((K, H), np.float32)
    sm[0, :len(vals)] = vals
    if K == 2:
        sm[1, :len(vals)] = vals[::-1]
    x = torch.ones((1, H), dtype=torch.bfloat16)
    ids = np.arange(K, dtype=np.int32)[None, :]
    pos = np.arange(K, dtype=np.int32)
    q = torch.zeros((K, H), dtype=torch.int8, device=dev())
    s = torch.zeros(K, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, s)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, K)
    assert s_ref[0] == sc32
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0
