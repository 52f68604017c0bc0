"""Continuous base-3 layout (five trits per byte across group boundaries, the
release summary's 1.72-bit accounting) against the oracle, through the C ABI
(needs a B200): bit-exact pack / unpack, and single-row products within the
bound |y - y_ref| <= 2e-3 * sum_k |w x'| + 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwht1024_b200 as bt
import workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0") if torch.cuda.is_available() else None
C = bt.LAYOUT_B3C


def T(a, dtype=None):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).to(DEV)
        return t.view(torch.bfloat16) if dtype == "bf16" else t
    return torch.from_numpy(a).to(DEV)


def check(y, y_ref, bound, extra=0.0):
    r = np.abs(y - y_ref) / (bound + extra)
    assert np.all(r <= 1.0), f"max err/bound {float(r.max()):.4g}"


@pytest.mark.parametrize("K", [128, 640, 1024, 5120, 17408])
def test_pack_unpack_bit_exact(K):
    g = workloads.rng(13000 + K)
    t = workloads.trits(g, 37, K)
    codes = bt.pack(T(t), C)
    ref = oracle.pack(t, oracle.LAYOUT_BASE3_CONT)
    assert np.array_equal(codes.cpu().numpy(), ref)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    back = bt.unpack(codes, K, C, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(back.cpu().numpy(), t)


def test_pack_worked_example_and_invalid_inputs():
    t = np.zeros((1, 1024), dtype=np.int8)
    t[0, :5] = [-1, 0, 1, -1, 1]
    codes = bt.pack(T(t), C)
    assert int(codes[0, 0].item()) == 183
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    bad = t.copy()
    bad[0, 700] = 3
    bt.pack(T(bad), C, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_TRIT
    c = oracle.pack(np.zeros((2, 128), dtype=np.int8), oracle.LAYOUT_BASE3_CONT)  # 26 bytes used of 32
    c[0, 3] = 250                     # not a base-3 code
    c[1, 25] = 121 - 27               # a pad trit that is not 0
    err.zero_()
    bt.unpack(T(c), 128, C, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_CODE and int(err.item()) & bt.DEVERR_INVALID_PAD
    c = oracle.pack(np.zeros((1, 128), dtype=np.int8), oracle.LAYOUT_BASE3_CONT)
    c[0, 30] = 1                      # row padding must be zero
    err.zero_()
    bt.unpack(T(c), 128, C, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_PAD


@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
@pytest.mark.parametrize("checked", [True, False])
def test_gemv_decode_triple_full_size(idx, layer, checked):
    case = workloads.layer_inputs("C1", layer, index=idx)
    codes = bt.pack(T(case["trits"]), C)
    err = torch.zeros(1, dtype=torch.int32, device=DEV) if checked else None
    y = bt.gemv(codes, T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), layer.N, C, dev_err=err)
    torch.cuda.synchronize()
    if checked:
        assert int(err.item()) == 0
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(y.cpu().numpy().astype(np.float64), y_ref, b)


@pytest.mark.parametrize("N,K", [(1, 1024), (17, 2048), (777, 3072), (300, 7168), (64, 76 * 1024)])
def test_gemv_ragged_shapes(N, K):
    # K % 640 != 0 for every K here: the last 640-column chunk is partial, and
    # chunks cross 1024-blocks; N = 1 and a ragged last row set
    case = workloads.random_case(13100 + N + K, 1, N, K)
    codes = bt.pack(T(case["trits"]), C)
    y = bt.gemv(codes, T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), N, C)
    torch.cuda.synchronize()
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(y.cpu().numpy().astype(np.float64), y_ref, b)


def test_gemv_prerotated_f32_and_bf16_out():
    g = workloads.rng(13200)
    N, K = 500, 3072
    t = workloads.trits(g, N, K)
    s = workloads.scales_f16_bits(g, N, K)
    x = g.standard_normal((1, K)).astype(np.float32)
    codes = bt.pack(T(t), C)
    y = bt.gemv(codes, T(s), T(x), None, N, C)                       # f32 x, no rotation
    yb = bt.gemv(codes, T(s), T(x), None, N, C, y_dtype=bt.BF16)
    torch.cuda.synchronize()
    y_ref, b = oracle.gemv(t, s, x.astype(np.float64))
    check(y.cpu().numpy().astype(np.float64), y_ref, b)
    yb64 = yb.float().cpu().numpy().astype(np.float64)
    a = np.abs(yb64)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8.0), 0.0)
    check(yb64, y_ref, b, half_ulp)


def test_gemv_zero_trits_and_group_straddling_bytes_exact():
    # all-zero rows give exactly 0; a single trit in a byte shared by two
    # groups (k = 128, byte 25 of the chunk) gives exactly s * x'_k
    case = workloads.random_case(13300, 1, 8, 2048)
    t = np.zeros_like(case["trits"])
    ks = [128, 256, 384, 512, 700, 1279, 1280]     # the split bytes' later trits, and chunk edges
    for r, k in enumerate(ks):
        t[r, k] = 1 if r % 2 == 0 else -1
    codes = bt.pack(T(t), C)
    y = bt.gemv(codes, T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), 8, C)
    torch.cuda.synchronize()
    # x' as the library computes it (bt_fwht1024 runs the same FP32 warp transform)
    xr = bt.fwht1024(T(case["x"], "bf16"), T(case["sign"]), bt.F32).cpu().numpy()
    yv = y.cpu().numpy()[0]
    assert yv[7] == 0.0
    for r, k in enumerate(ks):
        s = np.float32(case["scales"][r, k // 128].view(np.float16))
        want = np.float32(1 if r % 2 == 0 else -1) * (s * xr[0, k])
        assert yv[r] == want, (r, k, yv[r], want)


def test_batched_triple_and_chain():
    sign_np = workloads.sign1024()
    cases = [workloads.layer_inputs("C1", L, index=i) for i, L in enumerate(workloads.TRIPLE)]
    probs = [dict(codes=bt.pack(T(c["trits"]), C), scales=T(c["scales"]), x=T(c["x"], "bf16"),
                  y=torch.empty((1, c["N"]), device=DEV), N=c["N"], K=c["K"]) for c in cases]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ys = bt.gemv_batched(probs, T(sign_np), C, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for c, y in zip(cases, ys):
        _, y_ref, b = oracle.forward(c["trits"], c["scales"], c["x"], sign_np)
        check(y.cpu().numpy().astype(np.float64), y_ref, b)
    # chained: 5120 -> 5120 -> 17408 -> 5120, each bf16 output the next input
    g = workloads.rng(13400)
    layers = [(5120, 5120), (5120, 17408), (17408, 5120)]
    cs, ps = [], []
    for i, (K, N) in enumerate(layers):
        c = {"trits": workloads.trits(g, N, K), "scales": workloads.scales_f16_bits(g, N, K)}
        p = dict(codes=bt.pack(T(c["trits"]), C), scales=T(c["scales"]),
                 y=torch.empty((1, N), dtype=torch.bfloat16, device=DEV), N=N, K=K)
        if i == 0:
            c["x"] = workloads.activations_bf16_bits(g, 1, K, True)
            p["x"] = T(c["x"], "bf16")
        else:
            p["x_from"] = i - 1
        cs.append(c)
        ps.append(p)
    ys = bt.gemv_batched(ps, T(sign_np), C, y_dtype=bt.BF16)
    torch.cuda.synchronize()
    for l, (c, y) in enumerate(zip(cs, ys)):
        xb = c["x"] if l == 0 else ys[l - 1].view(torch.int16).cpu().numpy().view(np.uint16)
        y_ref, b = oracle.gemv(c["trits"], c["scales"], oracle.rotate_bf16(xb, sign_np))
        y64 = y.float().cpu().numpy().astype(np.float64)
        a = np.abs(y64)
        half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8.0), 0.0)
        check(y64, y_ref, b, half_ulp)
