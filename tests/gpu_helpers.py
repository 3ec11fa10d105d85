"""Shared helpers of the GPU parity tests: move data, run the CUDA path through the
binding, run the oracle on the same inputs."""
import numpy as np
import torch

import dispatch_combine_topk_b200 as mep
import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def dev():
    return torch.device("cuda", 0)


def gpu_plan_balanced(ids: np.ndarray, R, E, S, K):
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, np.int32).ravel()).to(dev())
    pb = mep.PlanBuffers.allocate(R, E, S, K, dev())
    mep.mep_plan(ids_d, R, E, S, K, pb)
    return pb


def gpu_plan_grouped(keys: np.ndarray, keep, R, n_keys, kpr, S, K):
    keys_d = torch.from_numpy(np.ascontiguousarray(keys, np.int32).ravel()).to(dev())
    keep_d = None if keep is None else torch.from_numpy(
        np.ascontiguousarray(keep, np.uint8).ravel()).to(dev())
    pb = mep.PlanBuffers.allocate(R, n_keys, S, K, dev())
    mep.mep_plan(keys_d, R, n_keys, S, K, pb, mode=mep.MEP_PLAN_GROUPED, keys_per_rank=kpr,
                 keep=keep_d)
    return pb


def assert_plan_equal(pb: "mep.PlanBuffers", p: "oracle.Plan", R: int):
    """Bit-exact comparison of every plan output with the oracle's."""
    assert np.array_equal(pb.pos.cpu().numpy(), p.pos), "pos"
    assert np.array_equal(pb.hist.cpu().numpy(), p.hist), "hist"
    assert np.array_equal(pb.rank_off.cpu().numpy(), p.rank_off), "rank_off"
    assert np.array_equal(pb.load.cpu().numpy(), p.load), "load"
    assert np.array_equal(pb.rep_count.cpu().numpy(), p.rep_count), "rep_count"
    assert np.array_equal(pb.rep_key.cpu().numpy(), p.rep_key), "rep_key"
    assert np.array_equal(pb.rep_cu.cpu().numpy(), p.rep_cu), "rep_cu"
    s = pb.stats_dict()
    assert (s["max_load"], s["max_chunk"], s["redundant"], s["prefetched"], s["n_kept"],
            s["max_hist"]) == (p.max_load, p.max_chunk, p.redundant, p.prefetched, p.n_kept,
                               p.max_hist)
    assert s["n_ranks_used"] == int((np.diff(p.rank_off) > 0).sum())
