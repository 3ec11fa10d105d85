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


def test_stream_synchronize_timeout_gives_up_then_sees_the_work_finish():
    """A host wait with a time limit on work that outlasts it: the wait reports the
    time-out, the work goes on, a later wait sees it finish, and the library still
    routes correctly afterwards."""
    torch.cuda.set_device(0)
    mep.mep_get_error(clear=True)
    f = mep.lib().mep_selftest_bounded_wait
    f.argtypes = [ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    s = torch.cuda.Stream(dev())
    flags = torch.full((8,), -1, dtype=torch.int32, device=dev())
    torch.cuda.synchronize()
    for i in range(8):       # each launch polls its barrier 2^22 times before giving up
        assert f(1 << 22, ctypes.c_void_p(flags[i:].data_ptr()), ctypes.c_void_p(s.cuda_stream)) == 0
    assert mep.mep_stream_synchronize_timeout(1, stream=s) is False
    assert mep.mep_stream_synchronize_timeout(120000, stream=s) is True
    assert flags.cpu().tolist() == [1] * 8
    assert mep.mep_get_error(clear=True) & MEP_DERR_TIMEOUT
    # an idle stream is done at once, and launches after a time-out still succeed
    assert mep.mep_stream_synchronize_timeout(0, stream=s) is True
    rng = np.random.default_rng(6)
    T, K, H = 20, 2, 64
    x = torch.randn((T, H), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    pos = rng.permutation(T * K).astype(np.int32)
    recv = torch.empty((T * K, H), dtype=torch.bfloat16, device=dev())
    with torch.cuda.stream(s):
        mep.mep_dispatch(x.to(dev()), torch.from_numpy(pos).to(dev()), K, recv, stream=s)
    assert mep.mep_stream_synchronize_timeout(60000, stream=s) is True
    assert np.array_equal(bits(recv), oracle.dispatch(bits(x), pos, K, T * K))
    assert mep.mep_get_error() == 0


def test_error_word_is_read_in_stream_order():
    """mep_get_error reads the word in order on the stream it is given, waiting for that
    stream only: a data error set by a kernel enqueued just before on the same stream is
    seen without any other synchronisation, and clearing it is ordered the same way."""
    torch.cuda.set_device(0)
    s = torch.cuda.Stream(dev())
    torch.cuda.synchronize()
    assert mep.mep_get_error(clear=True, stream=s) == 0
    T, K, H = 4, 2, 64
    x = torch.zeros((T, H), dtype=torch.bfloat16, device=dev())
    pos = torch.tensor([0, 1, 2, 3, 4, 5, 6, 99], dtype=torch.int32, device=dev())
    recv = torch.zeros((T * K, H), dtype=torch.bfloat16, device=dev())
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        mep.mep_dispatch(x, pos, K, recv, stream=s)
        assert mep.mep_get_error(clear=True, stream=s) == mep.DERR_ROW_RANGE
        assert mep.mep_get_error(clear=False, stream=s) == 0
