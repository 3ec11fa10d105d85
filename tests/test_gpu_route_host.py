"""One routing round trip from host memory through a single C call (mep_route_host):
the result equals the oracle routing the same tokens, and the device-side calls."""
import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
import synth
from gpu_helpers import bits, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_error_word():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    yield


def _host(w, pinned):
    ids, gates = synth.router(w)
    x = synth.hidden(w)
    t = [torch.from_numpy(ids).view(-1).contiguous(), torch.from_numpy(gates).view(-1).contiguous(), x.contiguous()]
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16)
    if pinned:
        t = [v.pin_memory() for v in t]
        out = out.pin_memory()
    return (*t, out)


@pytest.mark.parametrize("quant", [0, 1])
@pytest.mark.parametrize("pinned", [True, False])
def test_route_host_tiny_matches_oracle(quant, pinned):
    w = synth.get("tiny")
    ids_h, gates_h, x_h, out_h = _host(w, pinned)
    rb = mep.RouteBuffers.allocate(w.R, w.E, w.S, w.K, w.H, quant, dev())
    s = torch.cuda.Stream(dev())
    mep.mep_route_host(rb, ids_h, gates_h, x_h, out_h, stream=s)
    s.synchronize()
    ref = oracle.route_tokens(bits(x_h), np.ones((w.T, w.K), bool), gates_h.numpy().reshape(w.T, w.K), w.K, quant)
    assert np.array_equal(bits(out_h), ref)
    p = oracle.plan_balanced(ids_h.numpy(), w.R, w.E, w.S, w.K)
    assert np.array_equal(rb.plan.pos.cpu().numpy(), p.pos)
    assert mep.mep_get_error() == 0


def test_route_host_equals_device_calls_and_overlaps_buffer_sets():
    """Three buffer sets on three streams, round robin over six batches (the bench's
    end-to-end pattern): every downloaded result equals the device-side route."""
    w = synth.scaled(synth.get("r8"), S=256)
    sets = [mep.RouteBuffers.allocate(w.R, w.E, w.S, w.K, w.H, 0, dev()) for _ in range(3)]
    streams = [torch.cuda.Stream(dev()) for _ in range(3)]
    batches = []
    for i in range(6):
        ws = synth.scaled(w, seed=500 + i)
        ids, gates = synth.router(ws)
        x = synth.hidden(ws)
        h = [torch.from_numpy(ids).view(-1).contiguous().pin_memory(),
             torch.from_numpy(gates).view(-1).contiguous().pin_memory(), x.contiguous().pin_memory(),
             torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()]
        batches.append(h)
    for i, h in enumerate(batches):
        mep.mep_route_host(sets[i % 3], *h, stream=streams[i % 3])
    torch.cuda.synchronize()
    for ids_h, gates_h, x_h, out_h in batches:
        pb = mep.PlanBuffers.allocate(w.R, w.E, w.S, w.K, dev())
        ids_d, g_d, x_d = ids_h.to(dev()), gates_h.to(dev()), x_h.to(dev())
        mep.mep_plan(ids_d, w.R, w.E, w.S, w.K, pb)
        recv = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev())
        mep.mep_dispatch(x_d, pb.pos, w.K, recv)
        out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev())
        mep.mep_combine(recv, pb.pos, g_d, w.K, out)
        assert torch.equal(out.cpu().view(torch.int16), out_h.view(torch.int16))
    assert mep.mep_get_error() == 0


def test_route_host_reports_the_failing_step():
    w = synth.get("tiny")
    ids_h, gates_h, x_h, out_h = _host(w, False)
    rb = mep.RouteBuffers.allocate(w.R, w.E, w.S, w.K, w.H, 0, dev())
    cs = rb.c_struct()
    cs.E = w.E + 1                       # E % R != 0: mep_plan refuses (MEP_ERR_VALUE)
    with pytest.raises(mep.MepError) as e:
        mep.mep_route_host(rb, ids_h, gates_h, x_h, out_h, c_struct=cs)
    assert e.value.status == 4
    cs = rb.c_struct()
    cs.workspace_bytes = 8               # too small: MEP_ERR_WORKSPACE
    with pytest.raises(mep.MepError) as e:
        mep.mep_route_host(rb, ids_h, gates_h, x_h, out_h, c_struct=cs)
    assert e.value.status == 5
