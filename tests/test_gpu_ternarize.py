"""bt_ternarize (the offline weight path) against the oracle, through the C ABI
(needs a B200). Which trit and which FP16 scale each weight gets is an integer
result decided in FP64 by both sides in the same order of operations, so the
comparison is bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwht1024_b200 as bt
import workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _weights(seed, N, K, outliers=True):
    g = workloads.rng(seed)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    if outliers:
        pos = g.choice(N * K, size=max(1, N * K // 1000), replace=False)
        W.reshape(-1)[pos] *= 20.0
    return W


@pytest.mark.parametrize("N,K", [(1, 1024), (3, 2048), (77, 3072), (256, 5120), (5120, 5120)])
def test_ternarize_bit_exact(N, K):
    W = _weights(13000 + N + K, N, K)
    sign = workloads.sign1024()
    t, s = bt.ternarize(torch.from_numpy(W).to(DEV), torch.from_numpy(sign).to(DEV))
    torch.cuda.synchronize()
    t_ref, s_ref = oracle.ternarize(W.astype(np.float64), sign)
    assert np.array_equal(t.cpu().numpy(), t_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_ref)


def test_ternarize_special_groups():
    # a row of zeros (scale 0, zero trits) and a constructed exact ternary target
    sign = workloads.sign1024()
    W = _weights(13100, 4, 1024, outliers=False)
    W[1] = 0.0
    t, s = bt.ternarize(torch.from_numpy(W).to(DEV), torch.from_numpy(sign).to(DEV))
    t_ref, s_ref = oracle.ternarize(W.astype(np.float64), sign)
    assert np.array_equal(t.cpu().numpy(), t_ref) and np.all(t_ref[1] == 0)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_ref) and np.all(s_ref[1] == 0)


def test_offline_path_then_the_decode_product():
    # float W -> ternarise -> pack -> GEMV of a rotated activation: matches the
    # oracle on the ternarised weights, and approximates the float product
    N, K = 512, 2048
    W = _weights(13200, N, K)
    sign = workloads.sign1024()
    x = workloads.activations_bf16_bits(workloads.rng(13201), 1, K, True)
    t, s = bt.ternarize(torch.from_numpy(W).to(DEV), torch.from_numpy(sign).to(DEV))
    codes = bt.pack(t)
    y = bt.gemv(codes, s, torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16),
                torch.from_numpy(sign).to(DEV), N)
    torch.cuda.synchronize()
    trits, scales = t.cpu().numpy(), s.cpu().numpy().view(np.uint16)
    _, y_ref, bound = oracle.forward(trits, scales, x, sign)
    y64 = y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(y64 - y_ref) <= bound)
    y_float = oracle.bf16_to_f64(x) @ W.astype(np.float64).T   # W x without quantisation
    rel = np.linalg.norm(y64 - y_float) / np.linalg.norm(y_float)
    assert rel < 0.5, rel                                        # ternary weights: a coarse but faithful product
    print("relative error of the ternarised product", rel)
