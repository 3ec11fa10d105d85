"""GPU parity of the int8 dispatch with per-expert smoothing scales against the oracle
(codes and scales bit for bit), through both entry points: mep_dispatch_int8_smooth
(per token: H % 4 == 0 with up to 64 columns per thread, in groups of 4, takes the fused
kernel, all K slots of a token in one CTA; other H or alignments the scalar kernel) and
mep_dispatch_int8_smooth_grouped (the slots sorted by expert within chunks of tokens,
then quantised along that list, for H % 4 == 0 up to 8192 and aligned buffers; other
shapes fall back to the per-token kernels). The full int8 workload is compared whole,
one rank partition at a time, and with all-ones scales against the plain per-token int8
dispatch."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev, gpu_plan_balanced

pytestmark = pytest.mark.gpu

ENTRY = {"token": mep.mep_dispatch_int8_smooth, "grouped": mep.mep_dispatch_int8_smooth_grouped}


@pytest.mark.parametrize("entry", ["token", "grouped"])
@pytest.mark.parametrize("K", [1, 2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("H", [8, 12, 64, 4096, 4100, 7168, 12288, 16384, 16388, 20000, 32768, 32772, 7])
def test_smooth_dispatch_matches_oracle(K, H, entry):
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
    ENTRY[entry](x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("entry", ["token", "grouped"])
@pytest.mark.parametrize("K,H", [(2, 4096), (4, 7168), (8, 4096), (8, 12288), (8, 7168), (1, 64), (3, 520)])
def test_smooth_dispatch_many_tokens_per_cta(K, H, entry):
    """More tokens than CTAs resident on the GPU, so every CTA walks many tokens (and,
    sorted, several chunks of tokens: 2048 // K tokens each, the last one ragged);
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
    ENTRY[entry](x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("entry", ["token", "grouped"])
@pytest.mark.parametrize("x_off,q_off", [(4, 4), (4, 0), (0, 4), (1, 0), (0, 1)])
def test_smooth_dispatch_offset_buffers(x_off, q_off, entry):
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
    ENTRY[entry](xv, torch.from_numpy(ids).to(dev()).view(-1), torch.from_numpy(pos).to(dev()), K,
                                 torch.from_numpy(sm).to(dev()), qv, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(qv.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("entry", ["token", "grouped"])
def test_smooth_dispatch_bad_ids_and_rows_are_skipped_and_flagged(entry):
    T, K, H, E = 64, 4, 4096, 8
    rng = np.random.default_rng(5)
    x = torch.randn((T, H), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    pos = np.arange(T * K, dtype=np.int32)
    ids[3, 1] = E + 2                                      # expert out of range: slot skipped
    sm = np.ones((E, H), np.float32)
    q = torch.full((T * K + 1, H), 55, dtype=torch.int8, device=dev())
    sc = torch.full((T * K + 1,), 7.0, dtype=torch.float32, device=dev())
    ENTRY[entry](x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
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
    ENTRY[entry](x.to(dev()), torch.from_numpy(np.where(ids < E, ids, 0)).to(dev()).view(-1),
                                 torch.from_numpy(pos_bad).to(dev()), K, torch.from_numpy(sm).to(dev()), q[: T * K],
                                 sc[: T * K])
    assert mep.mep_get_error() & mep.DERR_ROW_RANGE


def test_smooth_dispatch_full_int8_workload():
    """The whole int8 workload through both entries: every code and scale against the
    oracle, one rank partition at a time; with all-ones scales, the plain per-token int8
    dispatch."""
    w = synth.get("int8")
    ids, _ = synth.router(w)
    x = synth.hidden(w)
    pb = gpu_plan_balanced(ids, w.R, w.E, w.S, w.K)
    x_d = x.to(dev())
    ids_d = torch.from_numpy(ids).to(dev()).view(-1)
    q = torch.empty((w.N, w.H), dtype=torch.int8, device=dev())
    sc = torch.empty(w.N, dtype=torch.float32, device=dev())
    q0 = torch.empty_like(q)
    s0 = torch.empty_like(sc)
    mep.mep_dispatch(x_d, pb.pos, w.K, q0, s0, quant=1)
    # all-ones scales: the plain per-token int8 dispatch, every row, through both entries
    ones = torch.ones((w.E, w.H), device=dev())
    for entry in ENTRY.values():
        q.fill_(0)
        entry(x_d, ids_d, pb.pos, w.K, ones, q, sc)
        assert torch.equal(q, q0) and torch.equal(sc.view(torch.int32), s0.view(torch.int32))
    del q0, s0, ones
    # per-expert scales: every slot of both entries against the oracle
    rng = np.random.default_rng(21)
    sm = (10.0 ** rng.uniform(-1, 1, (w.E, w.H))).astype(np.float32)
    sm_d = torch.from_numpy(sm).to(dev())
    mep.mep_dispatch_int8_smooth(x_d, ids_d, pb.pos, w.K, sm_d, q, sc)
    qg = torch.zeros_like(q)
    sg = torch.zeros_like(sc)
    mep.mep_dispatch_int8_smooth_grouped(x_d, ids_d, pb.pos, w.K, sm_d, qg, sg)
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
        for qq, ss in ((q, sc), (qg, sg)):
            assert np.array_equal(qq[lo:hi].cpu().numpy(), q_ref), r
            assert np.array_equal(ss[lo:hi].cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), r
        return r
    with ThreadPoolExecutor(8) as ex:
        assert sorted(ex.map(one, range(w.R))) == list(range(w.R))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("entry", ["token", "grouped"])
@pytest.mark.parametrize("K", [1, 2])
@pytest.mark.parametrize("amax", [381.0, 88.9, 1.0e-3, 5.0e30, 1.0e-36])
def test_quantiser_at_and_next_to_half_integer_quotients(amax, K, entry):
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
    ENTRY[entry](x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                 torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, s)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, K)
    assert s_ref[0] == sc32
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


@pytest.mark.parametrize("E", [6000, 6001])
def test_smooth_grouped_expert_count_limit(E):
    """Up to 6000 experts the grouped entry sorts the slots (the sort's counters fill its
    shared memory); past that it runs the per-token kernel. Same codes either way."""
    rng = np.random.default_rng(E)
    T, K, H = 300, 4, 64
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(E)) * 2).to(torch.bfloat16)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    ids[:40] = np.arange(E - K, E, dtype=np.int32)         # the last experts: the last counters
    rows = T * K
    pos = rng.permutation(rows).astype(np.int32)
    sm = (10.0 ** rng.uniform(-1, 1, (E, H))).astype(np.float32)
    q = torch.zeros((rows, H), dtype=torch.int8, device=dev())
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    mep.mep_dispatch_int8_smooth_grouped(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                         torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert mep.mep_get_error() == 0


def test_smooth_grouped_skewed_experts_and_long_runs():
    """Most slots on a few experts (runs of one expert much longer than a CTA's share of
    the sorted list, and CTAs whose slots change expert), several chunks of tokens."""
    rng = np.random.default_rng(77)
    T, K, H, E = 5000, 4, 1024, 64
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(77)) * 3).to(torch.bfloat16)
    w = 1.0 / np.arange(1, E + 1) ** 1.5
    ids = np.stack([rng.choice(E, K, replace=False, p=w / w.sum()) for _ in range(T)]).astype(np.int32)
    rows = T * K
    pos = rng.permutation(rows).astype(np.int32)
    pos[rng.random(rows) < 0.05] = -1
    sm = (10.0 ** rng.uniform(-1, 1, (E, H))).astype(np.float32)
    q = torch.zeros((rows, H), dtype=torch.int8, device=dev())
    sc = torch.zeros(rows, dtype=torch.float32, device=dev())
    ws = torch.empty(mep.mep_dispatch_int8_smooth_workspace_size(T, K), dtype=torch.uint8, device=dev())
    mep.mep_dispatch_int8_smooth_grouped(x.to(dev()), torch.from_numpy(ids).to(dev()).view(-1),
                                         torch.from_numpy(pos).to(dev()), K, torch.from_numpy(sm).to(dev()), q, sc,
                                         workspace=ws)
    q_ref, s_ref = oracle.dispatch_int8_smooth(bits(x), ids, pos, K, sm, rows)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    # the sorted list holds every slot once, each chunk's slots in expert order
    order = ws[: 4 * T * K].view(torch.int32).cpu().numpy()
    chunk = 2048 // K
    for c in range(0, T, chunk):
        lo, hi = c * K, min(T, c + chunk) * K
        part = order[lo:hi]
        assert np.array_equal(np.sort(part), np.arange(lo, hi))
        key = np.where(pos.reshape(-1)[part] >= 0, ids.reshape(-1)[part], E)
        assert np.all(np.diff(key) >= 0)
    assert mep.mep_get_error() == 0
