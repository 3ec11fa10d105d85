"""Failure handling on the GPU without faulting it.

A wait that nothing ends must run out, report MEP_DERR_TIMEOUT through the device
error word and leave the context usable; data errors are reported the same way (their
tests sit with the kernels they concern)."""
import ctypes

import numpy as np
import pytest
import torch

import dispatch_combine_topk_b200 as mep
import oracle
from gpu_helpers import bits, dev

pytestmark = pytest.mark.gpu

MEP_DERR_TIMEOUT = 0x10


def _selftest(max_polls):
    f = mep.lib().mep_selftest_bounded_wait
    f.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    flag = torch.full((1,), -1, dtype=torch.int32, device=dev())
    rc = f(max_polls, ctypes.c_void_p(flag.data_ptr()),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, int(flag.item())


def test_bounded_wait_runs_out_and_the_context_survives():
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    rc, timed_out = _selftest(20000)
    assert rc == 0 and timed_out == 1
    assert mep.mep_get_error(clear=True) & MEP_DERR_TIMEOUT
    # the context is still usable: a routing round trip still matches the oracle
    rng = np.random.default_rng(4)
    T, K, H = 40, 4, 256
    x = (torch.randn((T, H), generator=torch.Generator().manual_seed(4))).to(torch.bfloat16)
    pos = rng.permutation(T * K).astype(np.int32)
    gates = rng.random(T * K).astype(np.float32)
    recv = torch.empty((T * K, H), dtype=torch.bfloat16, device=dev())
    pos_d = torch.from_numpy(pos).to(dev())
    mep.mep_dispatch(x.to(dev()), pos_d, K, recv)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev())
    mep.mep_combine(recv, pos_d, torch.from_numpy(gates).to(dev()), K, out)
    y = oracle.dispatch(bits(x), pos, K, T * K)
    assert np.array_equal(bits(recv), y)
    assert np.array_equal(bits(out), oracle.combine(y, pos, gates, K))
    assert mep.mep_get_error() == 0


def test_selftest_arguments():
    f = mep.lib().mep_selftest_bounded_wait
    f.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    one = torch.zeros(1, dtype=torch.int32, device=dev())
    assert f(0, ctypes.c_void_p(one.data_ptr()), None) == 4
    assert f(10, None, None) == 1
