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
