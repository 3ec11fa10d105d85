"""The multi-rank host logic of bench.py on CPU with gloo, world_size 2: every rank
routes its own independent batch, the job time is the max over ranks, and the
reference arm prints from rank 0 only."""
import io
import os
import contextlib

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.scaled(synth.get("tiny"), S=16)
        wr = bench.rank_workload(w, rank)
        ids, _ = synth.router(wr)
        t = torch.from_numpy(ids.astype(np.int64)).view(-1)
        gathered = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        differ = not torch.equal(gathered[0], gathered[1])
        m = bench.max_over_ranks(1.5 + rank * 2.0, dist, torch.device("cpu"))
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            args = type("A", (), dict(steps=1, warmup=0, gpus=world, ref_div=4))()
            bench.run_reference(args, w)
        q.put((rank, differ, m, buf.getvalue(), wr.seed))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29000 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, d0, m0, out0, s0), (r1, d1, m1, out1, s1) = res
    assert d0 and d1                      # independent batches
    assert s0 != s1
    assert m0 == m1 == 3.5                # max over ranks
    assert '"impl": "reference"' in out0 and out1 == ""


def _ep_worker(rank, world, port, q):
    """One EP rank on CPU: its own slots of a shared workload, the plan's exchange step
    (all-gather of the per-rank histograms) through the package's orchestration, with the
    oracle standing in for the two device calls."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    import synth
    from dispatch_combine_topk_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.scaled(synth.get("tiny"), R=world, E=8 * world, S=96)
        ids_all, _ = synth.router(w)
        ids_all = ids_all.reshape(world, w.S * w.K)
        mine = torch.from_numpy(ids_all[rank].copy())
        seen = {}

        def histogram(i, n):
            return torch.from_numpy(oracle.histogram(i.numpy(), n).astype(np.int32))

        def plan(i, hist_all, R, E, S, K, r, out):
            seen.update(hist_all=hist_all.numpy().copy(), rank=r, R=R)
            return None

        ep.plan_rank(mine, w.E, w.S, w.K, histogram=histogram, plan=plan)
        direct = ep.gather_histograms(torch.full((5,), rank + 10, dtype=torch.int32))
        q.put((rank, seen["rank"], seen["R"], seen["hist_all"], direct.numpy(), ids_all))
    finally:
        dist.destroy_process_group()


def test_ep_histogram_exchange_two_gloo_ranks():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_ep_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    E = 16
    for rank, seen_rank, seen_R, hist_all, direct, ids_all in res:
        assert seen_rank == rank and seen_R == 2
        # row r of the gathered matrix is rank r's histogram, on every rank
        want = np.stack([oracle.histogram(ids_all[r], E) for r in range(2)])
        assert np.array_equal(hist_all, want)
        assert np.array_equal(direct, [[10] * 5, [11] * 5])
    assert np.array_equal(res[0][3], res[1][3])
