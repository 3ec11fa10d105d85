"""The routing step captured into a CUDA graph: replays on new inputs give the same
results as eager calls (balanced bf16, balanced int8, and the mapping op with the
grouped plan)."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import synth

pytestmark = pytest.mark.gpu


def _inputs(w, seed):
    ws = synth.scaled(w, seed=seed)
    ids, gates = synth.router(ws)
    return ids, gates, synth.hidden(ws)


@pytest.mark.parametrize("name,S", [("r8", 256), ("int8", 64), ("map", 256)])
def test_graph_replay_matches_eager(name, S):
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.scaled(synth.get(name), S=S)
    ids0, gates0, x0 = _inputs(w, 100)
    ids_d = torch.from_numpy(ids0).to(dev).view(-1)
    g_d = torch.from_numpy(gates0).to(dev).view(-1)
    x_d = x0.to(dev)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    if w.mapping:
        table, thr, active = synth.mapping_inputs(w)
        table_d, thr_d = torch.from_numpy(table).to(dev), torch.from_numpy(thr).to(dev)
        act_d = torch.from_numpy(active.astype(np.uint8)).to(dev)
        bids = torch.empty((w.T, w.K), dtype=torch.int32, device=dev)
        bmask = torch.empty((w.T, w.K), dtype=torch.uint8, device=dev)
        n_keys = w.R * w.place_per_rank
        pb = mep.PlanBuffers.allocate(w.R, n_keys, w.S, w.K, dev)
        recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    else:
        pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
        if w.quant:
            recv = torch.empty((w.N, w.H), dtype=torch.int8, device=dev)
            sc = torch.empty(w.N, dtype=torch.float32, device=dev)
            y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
        else:
            recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)

    def step(s):
        if w.mapping:
            for r in range(w.R):
                sl = slice(r * w.S, (r + 1) * w.S)
                mep.mep_update_expert(ids_d.view(w.T, w.K)[sl], table_d, g_d.view(w.T, w.K)[sl], thr_d,
                                      act_d[sl], r, w.R, 1, bids[sl], bmask[sl], stream=s)
            mep.mep_plan(bids.view(-1), w.R, n_keys, w.S, w.K, pb, mode=mep.MEP_PLAN_GROUPED,
                         keys_per_rank=w.place_per_rank, keep=bmask.view(-1), stream=s)
            mep.mep_dispatch(x_d, pb.pos, w.K, recv, stream=s)
            mep.mep_combine(recv, pb.pos, g_d, w.K, out, stream=s)
        else:
            mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb, stream=s)
            if w.quant:
                mep.mep_dispatch(x_d, pb.pos, w.K, recv, sc, quant=1, stream=s)
                mep.mep_dequantize(recv, sc, y, stream=s)
                mep.mep_combine(y, pb.pos, g_d, w.K, out, stream=s)
            else:
                mep.mep_dispatch(x_d, pb.pos, w.K, recv, stream=s)
                mep.mep_combine(recv, pb.pos, g_d, w.K, out, stream=s)

    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        step(s)                      # eager once first (one-time set-up happens here)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for seed in (200, 300):
        ids, gates, x = _inputs(w, seed)
        ids_d.copy_(torch.from_numpy(ids).view(-1))
        g_d.copy_(torch.from_numpy(gates).view(-1))
        x_d.copy_(x)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = [out.clone(), pb.pos.clone(), pb.rep_cu.clone(), pb.stats.clone()]
        with torch.cuda.stream(s):
            step(s)
        s.synchronize()
        want = [out, pb.pos, pb.rep_cu, pb.stats]
        for a, b in zip(got, want):
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b)
    del g
    assert mep.mep_get_error() == 0


def test_graph_replay_of_the_other_calls():
    """Histogram, int8 combine, the fused RMSNorm epilogue, the smooth-quantised
    dispatch, the prefetch plan and copy, and the gradient reduce, captured once and
    replayed on new inputs, equal eager calls."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.scaled(synth.get("r8"), S=128)
    B, D = w.E // w.R, 4096
    ids0, gates0, x0 = _inputs(w, 5)
    ids_d = torch.from_numpy(ids0).to(dev).view(-1)
    g_d = torch.from_numpy(gates0).to(dev).view(-1)
    x_d = x0.to(dev)
    smooth = torch.rand((w.E, w.H), device=dev) + 0.5
    res = torch.randn((w.T, w.H), device=dev).to(torch.bfloat16)
    gam = torch.ones(w.H, device=dev).to(torch.bfloat16)
    hist = torch.empty(w.E, dtype=torch.int32, device=dev)
    pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
    q = torch.empty((w.N, w.H), dtype=torch.int8, device=dev)
    sc = torch.empty(w.N, dtype=torch.float32, device=dev)
    recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    o1 = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    xo, yo = torch.empty_like(o1), torch.empty_like(o1)
    rstd = torch.empty(w.T, dtype=torch.float32, device=dev)
    se = torch.empty((w.R, B), dtype=torch.int32, device=dev)
    rw = torch.empty((w.R, w.E), dtype=torch.int32, device=dev)
    w_home = torch.randn((w.E, D), device=dev).to(torch.bfloat16)
    w_slots = torch.zeros((w.R * B, D), dtype=torch.bfloat16, device=dev)
    gh0 = torch.randn((w.E, D), device=dev)
    gs0 = torch.randn((w.R * B, D), device=dev)
    gh, gs = gh0.clone(), gs0.clone()

    def step(s):
        mep.mep_histogram(ids_d, w.E, hist, stream=s)
        mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb, stream=s)
        mep.mep_dispatch_int8_smooth(x_d, ids_d, pb.pos, w.K, smooth, q, sc, stream=s)
        mep.mep_combine_int8(q, sc, pb.pos, g_d, w.K, o1, stream=s)
        mep.mep_dispatch(x_d, pb.pos, w.K, recv, stream=s)
        mep.mep_combine_add_rmsnorm(recv, pb.pos, g_d, w.K, res, gam, 1e-6, xo, yo, rstd, stream=s)
        mep.mep_prefetch_plan(pb, w.R, w.E, B, se, rw, stream=s)
        mep.mep_prefetch_weights(w_home, se, w.R, B, w_slots, stream=s)
        mep.mep_grad_reduce(gh, gs, se, w.R, B, stream=s)

    outs = [hist, pb.pos, q, sc, o1, xo, yo, rstd, se, rw, w_slots, gh, gs]
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        step(s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for seed in (6, 7):
        ids, gates, x = _inputs(w, seed)
        ids_d.copy_(torch.from_numpy(ids).view(-1))
        g_d.copy_(torch.from_numpy(gates).view(-1))
        x_d.copy_(x)
        gh.copy_(gh0)
        gs.copy_(gs0)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in outs]
        gh.copy_(gh0)
        gs.copy_(gs0)
        with torch.cuda.stream(s):
            step(s)
        s.synchronize()
        for a, b in zip(got, outs):
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b)
    del g
    assert mep.mep_get_error() == 0


def test_graph_replay_of_the_deduplicated_dispatch():
    """Plan, dedup encoding, send, expand and combine captured once; replays on new
    inputs equal the plain eager route of those inputs."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = synth.scaled(synth.get("r8"), S=256)
    ids0, gates0, x0 = _inputs(w, 300)
    ids_d = torch.from_numpy(ids0).to(dev).view(-1)
    g_d = torch.from_numpy(gates0).to(dev).view(-1)
    x_d = x0.to(dev)
    pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
    db = mep.DedupBuffers.allocate(w.R, w.S, w.K, dev)
    sent = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)

    def step(s):
        mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb, stream=s)
        mep.mep_dedup_plan(pb.pos, pb.rank_off, w.R, w.S, w.K, db, stream=s)
        mep.mep_dispatch(x_d, db.dsend, w.K, sent, stream=s)
        mep.mep_expand(sent, db.gidx, recv, stream=s)
        mep.mep_combine(recv, pb.pos, g_d, w.K, out, stream=s)

    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        step(s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for seed in (301, 302):
        ids1, gates1, x1 = _inputs(w, seed)
        ids_d.copy_(torch.from_numpy(ids1).view(-1))
        g_d.copy_(torch.from_numpy(gates1).view(-1))
        x_d.copy_(x1)
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        got = out.clone()
        # plain eager route of the same inputs
        pb2 = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev)
        mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb2)
        recv2 = torch.empty_like(recv)
        mep.mep_dispatch(x_d, pb2.pos, w.K, recv2)
        out2 = torch.empty_like(out)
        mep.mep_combine(recv2, pb2.pos, g_d, w.K, out2)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), out2.view(torch.int16))
        assert torch.equal(recv.view(torch.int16), recv2.view(torch.int16))
    assert mep.mep_get_error() == 0
    del g
