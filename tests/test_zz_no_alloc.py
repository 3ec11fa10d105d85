"""mep_plan_static_ws: the plan entry point that allocates nothing.

Some callers cannot call cudaMalloc where they route tokens: a program whose device
memory is all owned by its own caching allocator or a fixed pool, a serving loop in
which an allocation could stall the device, a C program with no allocator for scratch.
For them the library keeps the plan's scratch in a 4 MiB array compiled into libmep.
These tests call that entry point through the C ABI and check that its plan equals, bit
for bit, the plan of mep_plan with a caller-provided workspace, on several calls in a
row with different shapes (leftovers of one call in the shared array would show up in
the next), and that it refuses a plan larger than its array.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import synth

pytestmark = pytest.mark.gpu

MEP_ERR_WORKSPACE = 5
STATIC_WS_BYTES = 4 << 20
FIELDS = ["pos", "hist", "rank_off", "load", "rep_count", "rep_key", "rep_cu", "stats"]


def _entry():
    f = mep.lib().mep_plan_static_ws
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_plan(ids_d, keep_d, R, n_keys, S, K, mode, kpr):
    """Outputs allocated by the test (pre-filled with a marker so that every word the
    call must write is checked), the plan computed by the C entry point."""
    dev = ids_d.device
    shapes = dict(pos=(R * S * K,), hist=(n_keys,), rank_off=(R + 1,), load=(R,), rep_count=(R,),
                  rep_key=(R, n_keys), rep_cu=(R, n_keys + 1), stats=(8,))
    out = {k: torch.full(v, -7, dtype=torch.int32, device=dev) for k, v in shapes.items()}
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _entry()(_p(ids_d), _p(keep_d), R, n_keys, S, K, mode, kpr, *[_p(out[k]) for k in FIELDS],
                  stream)
    torch.cuda.synchronize()
    return rc, out


def _cases():
    rng = np.random.default_rng(77)
    w = synth.get("r8")
    ids_r8, _ = synth.router(w)
    yield "r8 workload, balanced", ids_r8.ravel(), None, w.R, w.E, w.S, w.K, 0, 0
    R, E, S, K = 5, 40, 777, 6
    p = rng.zipf(1.3, E).astype(np.float64)
    ids = rng.choice(E, size=R * S * K, p=p / p.sum()).astype(np.int32)
    yield "ragged balanced", ids, None, R, E, S, K, 0, 0
    R, kpr, S, K = 4, 24, 1500, 8
    keys = rng.integers(0, R * kpr, R * S * K).astype(np.int32)
    keep = (rng.random(R * S * K) < 0.6).astype(np.uint8)
    yield "grouped with dropped slots", keys, keep, R, R * kpr, S, K, 1, kpr
    yield "r8 workload again", ids_r8.ravel(), None, w.R, w.E, w.S, w.K, 0, 0


def test_static_scratch_plan_equals_workspace_plan_on_calls_in_a_row():
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    mep.mep_get_error(clear=True)
    n = 0
    for name, ids, keep, R, n_keys, S, K, mode, kpr in _cases():
        ids_d = torch.from_numpy(ids).to(dev)
        keep_d = None if keep is None else torch.from_numpy(keep).to(dev)
        assert mep.mep_plan_workspace_size(R, n_keys, S, K) <= STATIC_WS_BYTES
        rc, got = _static_plan(ids_d, keep_d, R, n_keys, S, K, mode, kpr)
        assert rc == 0, (name, rc)
        ref = mep.PlanBuffers.allocate(R, n_keys, S, K, dev)
        mep.mep_plan(ids_d, R, n_keys, S, K, ref, mode=mode, keys_per_rank=kpr, keep=keep_d)
        torch.cuda.synchronize()
        for f in FIELDS:
            assert torch.equal(got[f], getattr(ref, f)), (name, f)
        n += 1
    assert n >= 2
    assert mep.mep_get_error() == 0


def test_static_scratch_plan_refuses_plans_larger_than_its_array():
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    R, n_keys, S, K = 8, 2048, 32768, 8          # 2^21 slots x 2048 keys: 8 MiB of scratch
    assert mep.mep_plan_workspace_size(R, n_keys, S, K) > STATIC_WS_BYTES
    one = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _entry()(_p(one), None, R, n_keys, S, K, 0, 0, *[_p(one)] * 8, stream)
    assert rc == MEP_ERR_WORKSPACE


def test_static_scratch_plan_after_a_device_reset(tmp_path):
    """The array's device address belongs to a CUDA context: after cudaDeviceReset the
    library must look it up again. A C program (its own process, so the reset cannot
    touch this one's context) plans with the static scratch and with a workspace, resets
    the device, and plans both ways twice more; every output must match bit for bit."""
    import os
    import subprocess
    from dispatch_combine_topk_b200 import build
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib = build.build()
    exe = tmp_path / "static_ws_reset"
    cuda = "/usr/local/cuda"
    subprocess.run(["gcc", "-O2", "-std=c11", os.path.join(root, "tests", "c", "static_ws_reset.c"),
                    "-I", os.path.join(root, "include"), "-I", os.path.join(cuda, "include"),
                    "-L", os.path.dirname(lib), "-lmep", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.join(cuda, "lib64"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "static_ws_reset ok" in r.stdout
