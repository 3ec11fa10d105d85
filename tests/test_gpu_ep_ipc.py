"""The expert-parallel exchange between processes: two processes, each one EP rank with
its own tokens and its own receive buffer, on one GPU, through ep.Exchange.

Each rank plans its own slots (its histogram, the all-gather of the histograms over a
gloo group, mep_plan_rank), maps the other rank's receive buffer into its process
through CUDA IPC, and dispatches its own token rows straight into both ranks' buffers
through the table of their addresses (mep_dispatch_ranks). After a fence every rank's
buffer must equal the oracle's dispatch restricted to that rank's partition of the
global plan, bit for bit, and each rank's combine over both buffers (mep_combine_ranks)
must equal the oracle's combine of its tokens. Two steps with different routings reuse
the buffers. No kernel waits on the other process: the processes meet only in host
barriers, with time limits."""
import datetime
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, quant, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import dispatch_combine_topk_b200 as mep
    from dispatch_combine_topk_b200 import ep
    import oracle
    import synth
    from gpu_helpers import bits
    result = {"rank": rank, "ok": False}
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        w = synth.scaled(synth.get("tiny"), R=world, E=8 * world, S=384, K=4, H=512)
        SK = w.S * w.K
        ex = ep.Exchange(w.E, w.S, w.K, w.H, quant=quant, device=dev)
        xb_all = None
        for step in range(2):
            ids_all, gates_all = synth.router(w)             # the whole batch, to check against
            if step == 1:                                    # another routing on the same buffers
                ids_all = np.ascontiguousarray(np.roll(ids_all.reshape(-1, w.K), 1, axis=1).reshape(ids_all.shape))
                ids_all = ((ids_all + 3) % w.E).astype(np.int32)
            x_all = synth.hidden(w)
            xb_all = bits(x_all)
            ids = torch.from_numpy(ids_all.reshape(world, SK)[rank].copy()).to(dev)
            rp, hist_all = ex.plan(ids)
            x = x_all[rank * w.S:(rank + 1) * w.S].to(dev)
            ex.dispatch(x, rp)
            ex.fence()                                       # every rank's rows are in place
            p = oracle.plan_balanced(ids_all, world, w.E, w.S, w.K)
            assert np.array_equal(rp.pos.cpu().numpy(), p.pos[rank * SK:(rank + 1) * SK]), "rows of this rank's slots"
            inside = (p.pos >= rank * SK) & (p.pos < (rank + 1) * SK)
            toks = np.unique(np.flatnonzero(inside) // w.K)
            pos_r = np.where(inside, p.pos - rank * SK, -1).astype(np.int32).reshape(-1, w.K)[toks]
            if quant:
                q_ref, s_ref = oracle.dispatch_int8(xb_all[toks], pos_r, w.K, SK)
                assert np.array_equal(ex.rows.cpu().numpy(), q_ref), "codes in this rank's buffer"
                assert np.array_equal(ex.scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
            else:
                assert np.array_equal(bits(ex.rows), oracle.dispatch(xb_all[toks], pos_r, w.K, SK)), "rows"
            # the identity expert leaves the rows as they are; every rank's outputs are final
            ex.fence()
            gates = torch.from_numpy(gates_all.reshape(world, SK)[rank].copy()).to(dev)
            out = torch.empty((w.S, w.H), dtype=torch.bfloat16, device=dev)
            ex.combine(rp, gates, out)
            torch.cuda.synchronize()
            pos_l = np.arange(SK, dtype=np.int32)
            xr = xb_all[rank * w.S:(rank + 1) * w.S]
            g = gates_all.reshape(world, SK)[rank]
            if quant:
                qq, ss = oracle.dispatch_int8(xr, pos_l, w.K, SK)
                ref = oracle.combine_int8(qq, ss, pos_l, g, w.K)
            else:
                ref = oracle.combine(oracle.dispatch(xr, pos_l, w.K, SK), pos_l, g, w.K)
            assert np.array_equal(bits(out), ref), f"combine, step {step}"
            assert hist_all.shape == (world, w.E)
            ex.fence()                                       # nobody reads a buffer the next step writes
        assert mep.mep_get_error() == 0
        ex.close()
        result["ok"] = True
    except Exception as e:                                   # reported to the parent
        result["error"] = repr(e)
    finally:
        try:
            dist.barrier()                                   # nobody unmaps a buffer still in use
        except Exception:
            pass
        q.put(result)
        dist.destroy_process_group()


@pytest.mark.parametrize("quant", [0, 1])
def test_two_processes_exchange_rows_through_ipc(quant):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + quant + os.getpid() % 200
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, quant, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=120)
    assert all(r["ok"] for r in res), res
    assert all(p.exitcode == 0 for p in procs)
