"""bt_gemv_noalloc: the GEMV for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they run the product: a custom
allocator or memory-pool callback, a runtime that has handed all device
memory to its own arena, or code held to a memory budget fixed in advance.
bt_gemv_noalloc takes the same inputs and outputs as bt_gemv but keeps its
scratch in a fixed array inside libbt.so. This file runs last (pytest
collects it last), so a run that stops at its first failure has already run
every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwht1024_b200 as bt
import workloads

pytestmark = pytest.mark.gpu


def _tensors(case, layout):
    dev = torch.device("cuda:0")
    codes = torch.from_numpy(oracle.pack(case["trits"], layout)).to(dev)
    scales = torch.from_numpy(case["scales"].view(np.int16)).to(dev)
    x = torch.from_numpy(case["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    sign = torch.from_numpy(case["sign"]).to(dev)
    return codes, scales, x, sign


# (1, 5120, 5120): the single-row kernel; (3, 1000, 3072): one TMA-fed launch;
# (9, 5120, 5120): two launches that reuse the scratch's counters and partials;
# (2, 1000, 3200): K not a multiple of 1024, pre-rotated FP32 x, the general
# register-fed kernel.
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M,N,K", [(1, 5120, 5120), (3, 1000, 3072), (9, 5120, 5120), (2, 1000, 3200)])
def test_noalloc_matches_workspace_entry_point(layout, M, N, K):
    case = workloads.random_case(7000 + M + layout, M, N, K)
    assert bt.gemv_workspace_bytes(layout, M, N, K) <= (8 << 20)
    codes, scales, x, sign = _tensors(case, layout)
    if K % 1024:
        xr = workloads.rng(7100 + M).standard_normal((M, K)).astype(np.float32)
        x, sign = torch.from_numpy(xr).to(x.device), None
        y_ref, bound = oracle.gemv(case["trits"], case["scales"], xr.astype(np.float64))
    else:
        _, y_ref, bound = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y_ws = bt.gemv(codes, scales, x, sign, N, layout).cpu().numpy().astype(np.float64)
    for _ in range(2):  # two calls in a row share (and reuse) the scratch array
        err = torch.zeros(1, dtype=torch.int32, device=x.device)
        y_na = bt.gemv_noalloc(codes, scales, x, sign, N, layout, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        y = y_na.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(y - y_ref) <= bound)          # the tolerance every GEMV test uses
        assert np.all(np.abs(y - y_ws) <= bound)
        assert np.array_equal(y, y_ws)                      # same kernels, deterministic order


def test_noalloc_rejects_requests_beyond_its_scratch():
    dev = torch.device("cuda:0")
    M, N, K = 16, 17408, 17408       # needs more than the 8 MiB built-in scratch
    assert bt.gemv_workspace_bytes(bt.LAYOUT_B3, M, N, K) > (8 << 20)
    codes = torch.zeros((N, bt.codes_row_bytes(bt.LAYOUT_B3, K)), dtype=torch.uint8, device=dev)
    scales = torch.zeros((N, K // 128), dtype=torch.int16, device=dev)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    with pytest.raises(bt.BtError) as e:
        bt.gemv_noalloc(codes, scales, x, None, N)
    assert e.value.status == 4  # BT_ERR_WORKSPACE, nothing launched
