"""bt_gemv_batched (the single-row decode over a list of matrices) against the
oracle, through the C ABI (needs a B200).

Independent matrices are compared element by element with the oracle's
y = W (R x). In a chain, layer l's input is layer l-1's output as the library
returned it (bf16), so every layer is checked against the oracle applied to
that same input: the per-layer bound |y - y_ref| <= 2e-3 * sum_k |w x'| + 1e-5,
plus half a bf16 ulp of the returned value where the output is bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_fwht1024_b200 as bt
import workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def T(a, dtype=None):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).to(DEV)
        return t.view(torch.bfloat16) if dtype == "bf16" else t
    return torch.from_numpy(a).to(DEV)


def bf16_half_ulp(y):
    a = np.abs(np.asarray(y, dtype=np.float64))
    out = np.zeros_like(a)
    nz = a > 0
    out[nz] = np.exp2(np.floor(np.log2(a[nz])) - 8.0)
    return out


def check(y, y_ref, bound, extra=0.0):
    r = np.abs(y - y_ref) / (bound + extra)
    assert np.all(r <= 1.0), f"max err/bound {float(r.max()):.4g}"
    return float(r.max())


def _weights(case, layout):
    return bt.pack(T(case["trits"]), layout), T(case["scales"])


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("checked", [True, False])
def test_batched_decode_triple(layout, checked):
    # the decode triple in one launch, each matrix with its own activation
    cases = [workloads.layer_inputs("C1", L, index=i) for i, L in enumerate(workloads.TRIPLE)]
    probs = []
    for c in cases:
        codes, sc = _weights(c, layout)
        probs.append(dict(codes=codes, scales=sc, x=T(c["x"], "bf16"), y=torch.empty((1, c["N"]), device=DEV),
                          N=c["N"], K=c["K"]))
    err = torch.zeros(1, dtype=torch.int32, device=DEV) if checked else None
    ys = bt.gemv_batched(probs, T(cases[0]["sign"]), layout, dev_err=err)
    torch.cuda.synchronize()
    if checked:
        assert int(err.item()) == 0
    for c, y in zip(cases, ys):
        _, y_ref, b = oracle.forward(c["trits"], c["scales"], c["x"], c["sign"])
        check(y.cpu().numpy().astype(np.float64), y_ref, b)


def test_batched_equals_single_calls_and_is_deterministic():
    cases = [workloads.layer_inputs("C1", L, index=i) for i, L in enumerate(workloads.TRIPLE)]
    sign = T(cases[0]["sign"])
    probs, singles = [], []
    for c in cases:
        codes, sc = _weights(c, bt.LAYOUT_B3)
        x = T(c["x"], "bf16")
        probs.append(dict(codes=codes, scales=sc, x=x, y=torch.empty((1, c["N"]), device=DEV), N=c["N"], K=c["K"]))
        singles.append(bt.gemv(codes, sc, x, sign, c["N"]))
    a = [y.clone() for y in bt.gemv_batched(probs, sign)]
    b = [y.clone() for y in bt.gemv_batched(probs, sign)]
    torch.cuda.synchronize()
    for ya, yb, ys in zip(a, b, singles):
        assert torch.equal(ya, yb)          # repeated calls: bit for bit
        assert torch.equal(ya, ys)          # a tile's result does not depend on the schedule


def _chain(layers, layout, seed, y_dtype=bt.BF16):
    """Problems of a chain: layer 0 takes a seeded activation, layer l > 0 the
    output of layer l - 1."""
    g = workloads.rng(seed)
    cases, probs = [], []
    for i, (K, N) in enumerate(layers):
        c = {"K": K, "N": N, "trits": workloads.trits(g, N, K), "scales": workloads.scales_f16_bits(g, N, K)}
        codes, sc = _weights(c, layout)
        y = torch.empty((1, N), dtype=torch.bfloat16 if y_dtype == bt.BF16 else torch.float32, device=DEV)
        p = dict(codes=codes, scales=sc, y=y, N=N, K=K)
        if i == 0:
            c["x"] = workloads.activations_bf16_bits(g, 1, K, True)
            p["x"] = T(c["x"], "bf16")
        else:
            p["x_from"] = i - 1
        cases.append(c)
        probs.append(p)
    return cases, probs


def _check_chain(cases, ys, sign_np, y_dtype=bt.BF16):
    x_bits = cases[0]["x"]
    worst = 0.0
    for l, (c, y) in enumerate(zip(cases, ys)):
        if y_dtype == bt.BF16:
            y64 = y.float().cpu().numpy().astype(np.float64)
        else:
            y64 = y.cpu().numpy().astype(np.float64)
        if l == 0:
            xr = oracle.rotate_bf16(x_bits, sign_np)
        else:
            prev = ys[l - 1]
            if y_dtype == bt.BF16:
                xb = prev.view(torch.int16).cpu().numpy().view(np.uint16)
                xr = oracle.rotate_bf16(xb, sign_np)
            else:
                xr = oracle.rotate(prev.cpu().numpy().astype(np.float64), sign_np)
        y_ref, b = oracle.gemv(c["trits"], c["scales"], xr)
        extra = bf16_half_ulp(y64) if y_dtype == bt.BF16 else 0.0
        worst = max(worst, check(y64, y_ref, b, extra))
    return worst


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_batched_chained_triples(layout):
    # two layer triples chained 5120 -> 5120 -> 17408 -> 5120 -> 5120 -> 17408 -> 5120:
    # each layer rotates the previous layer's bf16 output inside the same launch
    layers = [(5120, 5120), (5120, 17408), (17408, 5120)] * 2
    cases, probs = _chain(layers, layout, 12000 + layout)
    sign_np = workloads.sign1024()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ys = bt.gemv_batched(probs, T(sign_np), layout, y_dtype=bt.BF16, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_chain(cases, ys, sign_np)


def test_batched_chain_across_launches():
    # 26 chained layers: three launches of at most 12, the links between them kept by stream order
    layers = [(2048, 2048)] * 26
    cases, probs = _chain(layers, bt.LAYOUT_B3, 12100)
    sign_np = workloads.sign1024()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ys = bt.gemv_batched(probs, T(sign_np), bt.LAYOUT_B3, y_dtype=bt.BF16, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_chain(cases, ys, sign_np)


def test_batched_chain_f32_prerotated():
    # no sign vector: every x is already rotated; FP32 outputs feed the next layer as they are
    layers = [(1024, 3072), (3072, 1024), (1024, 777)]
    g = workloads.rng(12200)
    cases, probs = [], []
    for i, (K, N) in enumerate(layers):
        c = {"K": K, "N": N, "trits": workloads.trits(g, N, K), "scales": workloads.scales_f16_bits(g, N, K)}
        codes, sc = _weights(c, bt.LAYOUT_B3)
        p = dict(codes=codes, scales=sc, y=torch.empty((1, N), device=DEV), N=N, K=K)
        if i == 0:
            c["x"] = g.standard_normal((1, K)).astype(np.float32)
            p["x"] = torch.from_numpy(c["x"]).to(DEV)
        else:
            p["x_from"] = i - 1
        cases.append(c)
        probs.append(p)
    ys = bt.gemv_batched(probs, None, bt.LAYOUT_B3, y_dtype=bt.F32)
    torch.cuda.synchronize()
    xin = cases[0]["x"].astype(np.float64)
    for l, (c, y) in enumerate(zip(cases, ys)):
        xr = xin if l == 0 else ys[l - 1].cpu().numpy().astype(np.float64)
        y_ref, b = oracle.gemv(c["trits"], c["scales"], xr)
        check(y.cpu().numpy().astype(np.float64), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("N,K", [(1, 1024), (17, 2048), (1000, 1024), (77, 76 * 1024), (300, 3072)])
def test_batched_ragged_and_edge_shapes(layout, N, K):
    # one row, a ragged last set, one 1024-block per row, a long row (152
    # chunks: more chunks than CTAs, so CTAs cover several chunks) and a
    # list of one
    case = workloads.random_case(12300 + N + K, 1, N, K)
    codes, sc = _weights(case, layout)
    y = torch.empty((1, N), device=DEV)
    bt.gemv_batched([dict(codes=codes, scales=sc, x=T(case["x"], "bf16"), y=y, N=N, K=K)], T(case["sign"]),
                    layout)
    torch.cuda.synchronize()
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(y.cpu().numpy().astype(np.float64), y_ref, b)


def test_batched_many_small_matrices_one_launch():
    # twelve independent matrices of different shapes in one launch: segments
    # of several matrices share CTAs
    shapes = [(1024, 64), (2048, 333), (1024, 1), (3072, 1500), (1024, 257), (5120, 100),
              (2048, 2048), (1024, 16), (4096, 999), (1024, 4000), (2048, 31), (1024, 512)]
    sign_np = workloads.sign1024()
    cases, probs = [], []
    for i, (K, N) in enumerate(shapes):
        c = workloads.random_case(12500 + i, 1, N, K)
        codes, sc = _weights(c, bt.LAYOUT_B3)
        probs.append(dict(codes=codes, scales=sc, x=T(c["x"], "bf16"), y=torch.empty((1, N), device=DEV), N=N, K=K))
        cases.append(c)
    ys = bt.gemv_batched(probs, T(sign_np))
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        _, y_ref, b = oracle.forward(c["trits"], c["scales"], c["x"], sign_np)
        check(y.cpu().numpy().astype(np.float64), y_ref, b)


def test_batched_zero_weights_exact_and_invalid_codes_flagged():
    # zero trits: every table entry is an exact 0 and integer sums of zeros stay 0
    K, N = 2048, 64
    case = workloads.random_case(12400, 1, N, K)
    sign = T(case["sign"])
    z = np.zeros_like(case["trits"])
    codes = bt.pack(T(z))
    y = torch.empty((1, N), device=DEV)
    bt.gemv_batched([dict(codes=codes, scales=T(case["scales"]), x=T(case["x"], "bf16"), y=y, N=N, K=K)], sign)
    torch.cuda.synchronize()
    assert torch.all(y == 0)                      # zero trits cancel exactly
    bad = oracle.pack(case["trits"])
    bad[9, 40] = 247
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    bt.gemv_batched([dict(codes=T(bad), scales=T(case["scales"]), x=T(case["x"], "bf16"), y=y, N=N, K=K)], sign,
                    dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_CODE
    assert torch.isfinite(y).all()


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_batched_outputs_feeding_later_matrices(layout):
    # inputs from the previous group (summed from its partials inside the next
    # kernel), from a group two launches back (read from memory) and given
    # activations, mixed in one list: groups {A}, {B, C}, {D, E, F}
    spec = [(1024, 2048, None), (2048, 1024, 0), (2048, 3072, 0), (1024, 1024, 1), (2048, 777, 0), (3072, 500, None)]
    g = workloads.rng(12600 + layout)
    sign_np = workloads.sign1024()
    cases, probs = [], []
    for K, N, src in spec:
        c = {"K": K, "N": N, "trits": workloads.trits(g, N, K), "scales": workloads.scales_f16_bits(g, N, K),
             "src": src}
        codes, sc = _weights(c, layout)
        p = dict(codes=codes, scales=sc, y=torch.empty((1, N), dtype=torch.bfloat16, device=DEV), N=N, K=K)
        if src is None:
            c["x"] = workloads.activations_bf16_bits(g, 1, K, True)
            p["x"] = T(c["x"], "bf16")
        else:
            p["x_from"] = src
        cases.append(c)
        probs.append(p)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ys = bt.gemv_batched(probs, T(sign_np), layout, y_dtype=bt.BF16, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for c, y in zip(cases, ys):
        xb = c["x"] if c["src"] is None else ys[c["src"]].view(torch.int16).cpu().numpy().view(np.uint16)
        y_ref, b = oracle.gemv(c["trits"], c["scales"], oracle.rotate_bf16(xb, sign_np))
        y64 = y.float().cpu().numpy().astype(np.float64)
        check(y64, y_ref, b, bf16_half_ulp(y64))
