"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Packing is compared byte for byte. Floating-point results are compared
element by element against the oracle's FP64 values with the acceptance
bound |y - y_ref| <= 2e-3 * sum_k |w x'| + 1e-5 (FP32 accumulation); the
rotation against |x' - x'_ref| <= 1e-6 * sum_j |x_j| / 32 + 1e-7 per element
(ten FP32 butterfly stages), plus half an ulp of bf16 when it rounds to bf16.
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


def f64(t):
    return t.float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else t.cpu().numpy().astype(np.float64)


def err_ratio(y, y_ref, bound):
    return float(np.max(np.abs(y - y_ref) / bound))


# ---------------------------------------------------------------- pack ----

@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("N,K", [(256, 1024), (5120, 5120), (77, 384), (1, 128), (3, 17408)])
def test_pack_unpack_bit_exact(layout, N, K):
    t = workloads.trits(workloads.rng(N * 7 + K), N, K)
    codes = bt.pack(T(t), layout)
    ref = oracle.pack(t, layout)
    assert np.array_equal(codes.cpu().numpy(), ref)
    back = bt.unpack(codes, K, layout)
    assert np.array_equal(back.cpu().numpy(), t)


def test_pack_exhaustive_codes():
    import itertools
    tuples = list(itertools.product((-1, 0, 1), repeat=5))
    t = np.zeros((len(tuples), 128), dtype=np.int8)
    for r, tup in enumerate(tuples):
        t[r, :5] = tup
        t[r, 125:128] = tup[:3]
    codes = bt.pack(T(t))
    assert np.array_equal(codes.cpu().numpy(), oracle.pack(t))
    assert int(codes[tuples.index((-1, 0, 1, -1, 1)), 0]) == 183


def test_pack_flags_invalid_trits():
    t = np.zeros((4, 256), dtype=np.int8)
    t[2, 77] = 3
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    codes = bt.pack(T(t), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_TRIT
    assert np.array_equal(codes.cpu().numpy(), oracle.pack(np.zeros_like(t)))


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_unpack_flags_invalid_codes(layout):
    t = workloads.trits(workloads.rng(5), 3, 256)
    codes = oracle.pack(t, layout)
    bad = codes.copy()
    bad[1, 7] = 250 if layout == bt.LAYOUT_B3 else 0xFF
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    bt.unpack(T(bad), 256, layout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_CODE
    if layout == bt.LAYOUT_B3:
        pad = codes.copy()
        pad[0, 25] = 0        # pad digits 0 -> non-zero pad trits
        err.zero_()
        bt.unpack(T(pad), 256, layout, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) & bt.DEVERR_INVALID_PAD


# ---------------------------------------------------------------- FWHT ----

@pytest.mark.parametrize("M,K", [(1, 1024), (1, 5120), (16, 17408), (512, 5120), (3, 2048)])
@pytest.mark.parametrize("out_dtype", [bt.F32, bt.BF16])
def test_fwht_vs_oracle(M, K, out_dtype):
    xb = workloads.fwht_input(M * 31 + K, M, K)
    s = workloads.sign1024()
    out = bt.fwht1024(T(xb, "bf16"), T(s), out_dtype)
    torch.cuda.synchronize()
    ref = oracle.rotate_bf16(xb, s)
    x = oracle.bf16_to_f64(xb).reshape(M, K // 1024, 1024)
    tol = 1e-6 * np.repeat(np.abs(x).sum(axis=2) / 32.0, 1024, axis=1).reshape(M, K) + 1e-7
    if out_dtype == bt.BF16:
        tol = tol + np.abs(ref) * 2.0 ** -8
    got = f64(out)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) / tol))


def test_fwht_matrix_form_small():
    xb = workloads.fwht_input(3, 2, 1024)
    s = workloads.sign1024()
    got = f64(bt.fwht1024(T(xb, "bf16"), T(s), bt.F32))
    ref = oracle.rotate(oracle.bf16_to_f64(xb), s, "matrix")
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


# ---------------------------------------------------------------- GEMV ----

def run_gemv(case, layout=bt.LAYOUT_B3, rotate=True, y_dtype=bt.F32, x_f32=None):
    codes = bt.pack(T(case["trits"]), layout)
    if rotate:
        x = T(case["x"], "bf16")
        sign = T(case["sign"])
    else:
        x = torch.from_numpy(x_f32.astype(np.float32)).to(DEV)
        sign = None
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = bt.gemv(codes, T(case["scales"]), x, sign, case["N"], layout, y_dtype, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return f64(y)


def check(y, y_ref, bound, extra=0.0):
    r = np.abs(y - y_ref) / (bound + extra)
    assert np.all(r <= 1.0), f"max err/bound {float(r.max()):.4g}"
    return float(r.max())


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_tiny_config(layout):
    case = workloads.layer_inputs("C0", workloads.TINY)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout), y_ref, b)


@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemv_decode_triple_full_size(idx, layer):
    case = workloads.layer_inputs("C1", layer, index=idx)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16])
def test_gemv_ragged_and_batched(layout, M):
    case = workloads.random_case(1000 + M, M, 1000, 3072)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("N,K", [(77, 1152), (16, 128), (33, 896), (5, 17408)])
def test_gemv_prerotated_ragged_groups(layout, N, K):
    case = workloads.random_case(2000 + N, 2, N, K)
    xr = workloads.rng(3000 + N).standard_normal((2, K)) * 3.0
    xr32 = xr.astype(np.float32).astype(np.float64)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr32)
    check(run_gemv(case, layout, rotate=False, x_f32=xr32), y_ref, b)


# Single-row (M = 1) calls with K % 1024 == 0 take the table-lookup kernel:
# one K chunk of 512 per CTA and row slices, or, with more chunks than SMs,
# CTAs that walk chunks. These cases cover its branches.

@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("N,K", [(1, 1024), (3, 2048), (17, 1024), (77, 3072), (1000, 17408)])
def test_gemv_m1_prerotated_f32(layout, N, K):
    case = workloads.random_case(2400 + N + K, 1, N, K)
    xr = workloads.rng(2500 + N).standard_normal((1, K)) * 3.0
    xr32 = xr.astype(np.float32).astype(np.float64)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr32)
    check(run_gemv(case, layout, rotate=False, x_f32=xr32), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_m1_prerotated_bf16(layout):
    N, K = 300, 5120
    case = workloads.random_case(2600, 1, N, K)
    xbits = workloads.activations_bf16_bits(workloads.rng(2601), 1, K, True)
    xr = oracle.bf16_to_f64(xbits)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    codes = bt.pack(T(case["trits"]), layout)
    y = bt.gemv(codes, T(case["scales"]), T(xbits, "bf16"), None, N, layout)
    check(f64(y), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_m1_walks_chunks(layout):
    # 76 blocks = 152 chunks of 512: more chunks than SMs, so CTAs walk chunks
    N, K = 40, 76 * 1024
    case = workloads.random_case(2700, 1, N, K)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_m1_bf16_output(layout):
    case = workloads.random_case(2800, 1, 5120, 5120)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemv(case, layout, y_dtype=bt.BF16)
    check(y, y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


def test_gemv_bf16_output():
    case = workloads.random_case(4000, 4, 512, 2048)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemv(case, y_dtype=bt.BF16)
    check(y, y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


def test_gemv_special_cases():
    case = workloads.random_case(5000, 1, 64, 2048)
    case["trits"] = np.zeros_like(case["trits"])
    y0 = run_gemv(case)
    assert np.all(np.abs(y0) <= 1e-5)
    case["trits"][17, 1500] = 1
    xr, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y1 = run_gemv(case)
    check(y1, y_ref, b)


def test_gemv_deterministic():
    case = workloads.layer_inputs("C1", workloads.TRIPLE[0], index=0)
    a = run_gemv(case)
    b = run_gemv(case)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_flags_invalid_codes(layout):
    case = workloads.random_case(6000, 1, 64, 1024)
    codes = oracle.pack(case["trits"], layout)
    codes[9, 40] = 247 if layout == bt.LAYOUT_B3 else 0xC3
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = bt.gemv(T(codes), T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), 64, layout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_CODE
    assert torch.isfinite(y).all()


# ---------------------------------------------------------------- GEMM ----

def run_gemm(trits, scales, x_bits, sign, layout=bt.LAYOUT_B3, x_f32=None):
    codes = bt.pack(T(trits), layout)
    if x_f32 is None:
        x = T(x_bits, "bf16")
        sg = T(sign)
    else:
        x = torch.from_numpy(x_f32.astype(np.float32)).to(DEV)
        sg = None
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = bt.gemm(codes, T(scales), x, sg, trits.shape[0], layout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return f64(y)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M,N,K", [(128, 256, 1024), (256, 384, 2048), (128, 128, 3072)])
def test_gemm_small_full(layout, M, N, K):
    case = workloads.random_case(8000 + N + K, M, N, K)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], layout)
    check(y, y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemm_prefill_triple_sampled_rows(idx, layer):
    # the pp512 shapes at full N and K; the oracle computes 8 sampled rows of Y
    case = workloads.layer_inputs("C3", layer, index=idx)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"])
    rows = np.sort(workloads.rng(9000 + idx).choice(512, size=8, replace=False))
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check(y[rows], y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


def test_gemm_2bit_prefill_shape_sampled():
    layer = workloads.TRIPLE[0]
    case = workloads.layer_inputs("C4", layer, M=512, index=0)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], bt.LAYOUT_2BIT)
    rows = np.array([0, 77, 300, 511])
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check(y[rows], y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


@pytest.mark.parametrize("M", [128, 256])   # 256: CTA pairs
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemm_prerotated_ragged_blocks(layout, M):
    # K = 1152: an odd number of K groups, and rows only 2-byte aligned
    N, K = 256, 1152
    case = workloads.random_case(8500, M, N, K)
    xr = workloads.rng(8501).standard_normal((M, K)) * 2.0
    xr32 = xr.astype(np.float32).astype(np.float64)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr32)
    y = run_gemm(case["trits"], case["scales"], None, None, layout, x_f32=xr32)
    check(y, y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


@pytest.mark.parametrize("M", [128, 256])
def test_gemm_special_cases(M):
    N, K = 128, 1024
    case = workloads.random_case(8600, M, N, K)
    z = np.zeros_like(case["trits"])
    y0 = run_gemm(z, case["scales"], case["x"], case["sign"])
    assert np.all(y0 == 0)
    z[3, 999] = -1
    _, y_ref, b = oracle.forward(z, case["scales"], case["x"], case["sign"])
    y1 = run_gemm(z, case["scales"], case["x"], case["sign"])
    check(y1, y_ref, b, extra=np.abs(y_ref) * 2.0 ** -8)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_unchecked_equals_checked(layout):
    # without an error word the code check is compiled out; results must not change
    case = workloads.layer_inputs("C1", workloads.TRIPLE[2], index=2)
    codes = bt.pack(T(case["trits"]), layout)
    x, sign, sc = T(case["x"], "bf16"), T(case["sign"]), T(case["scales"])
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    a = bt.gemv(codes, sc, x, sign, case["N"], layout, dev_err=err)
    b = bt.gemv(codes, sc, x, sign, case["N"], layout)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(a, b)
