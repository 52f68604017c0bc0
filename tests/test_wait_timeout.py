"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait in libbt.so is bounded (a number of tries, or a time on the global
timer); one that runs out sets BT_DEVERR_TIMEOUT in the caller's error word,
lets the copies still in flight land and returns, so the context stays
usable. These tests load the test-only twin of the library
(libbt_waittest.so), in which the single-row kernel never requests one set of
rows -- the second set of CTA 0's warp 0 -- and every wait gives up after
20 ms. They check that the call returns with the timeout bit set, that a
second timed-out call behaves the same, and that the product library still
matches the oracle in the same process. Nothing traps, faults or spins
without a bound.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwht1024_b200 as bt
import workloads
from ternary_weight_fwht1024_b200 import _build

pytestmark = pytest.mark.gpu


def _waittest_lib():
    lib = ctypes.CDLL(_build.build_waittest())
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.bt_gemv_workspace_bytes.argtypes = [I, I64, I64, I64]
    lib.bt_gemv_workspace_bytes.restype = SZ
    lib.bt_gemv.argtypes = [I, P, P, P, I, P, I64, I64, I64, I, P, P, SZ, P, P]
    lib.bt_gemv.restype = I
    return lib


def test_withheld_copy_times_out_and_the_context_survives():
    dev = torch.device("cuda:0")
    # 152 chunks of 512: CTA 0's share is the 1000 rows of chunk 0, so its
    # warp 0 streams sets 0, 16, 32 and 48 and the second of them is left out
    N, K = 1000, 76 * 1024
    case = workloads.random_case(11000, 1, N, K)
    codes = bt.pack(torch.from_numpy(case["trits"]).to(dev))
    scales = torch.from_numpy(case["scales"].view(np.int16)).to(dev)
    x = torch.from_numpy(case["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    sign = torch.from_numpy(case["sign"]).to(dev)
    y = torch.empty((1, N), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    lib = _waittest_lib()
    need = lib.bt_gemv_workspace_bytes(bt.LAYOUT_B3, 1, N, K)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = lib.bt_gemv(bt.LAYOUT_B3, vp(codes), vp(scales), vp(x), bt.BF16, vp(sign), 1, N, K, bt.F32, vp(y),
                     vp(ws), need, vp(err), stream)
    assert st == 0
    torch.cuda.synchronize()                      # the kernel returned
    assert int(err.item()) & bt.DEVERR_TIMEOUT
    assert not int(err.item()) & bt.DEVERR_INVALID_CODE

    # the context is still usable: the product library gives the oracle's result
    _, y_ref, bound = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    err.zero_()
    y2 = bt.gemv(codes, scales, x, sign, N, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.all(np.abs(y2.cpu().numpy().astype(np.float64) - y_ref) <= bound)


def test_withheld_copy_twice_then_a_correct_call():
    dev = torch.device("cuda:0")
    N, K = 17408, 5120         # CTA 0's share: over 900 rows of chunk 0, so warp 0 has sets 0, 16, 32, ...
    case = workloads.random_case(11100, 1, N, K)
    codes = bt.pack(torch.from_numpy(case["trits"]).to(dev))
    scales = torch.from_numpy(case["scales"].view(np.int16)).to(dev)
    x = torch.from_numpy(case["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    sign = torch.from_numpy(case["sign"]).to(dev)
    y = torch.empty((1, N), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    lib = _waittest_lib()
    need = lib.bt_gemv_workspace_bytes(bt.LAYOUT_B3, 1, N, K)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=dev)  # the workspace's contents do not matter
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for _ in range(2):
        err.zero_()
        st = lib.bt_gemv(bt.LAYOUT_B3, vp(codes), vp(scales), vp(x), bt.BF16, vp(sign), 1, N, K, bt.F32, vp(y),
                         vp(ws), need, vp(err), stream)
        assert st == 0
        torch.cuda.synchronize()
        assert int(err.item()) & bt.DEVERR_TIMEOUT

    _, y_ref, bound = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    err.zero_()
    y2 = bt.gemv(codes, scales, x, sign, N, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.all(np.abs(y2.cpu().numpy().astype(np.float64) - y_ref) <= bound)
