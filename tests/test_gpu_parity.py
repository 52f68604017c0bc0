"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Packing is compared byte for byte. Floating-point results are compared
element by element against the oracle's FP64 values with the acceptance
bound |y - y_ref| <= 2e-3 * sum_k |w x'| + 1e-5 (FP32 accumulation); the
rotation against |x' - x'_ref| <= 1e-6 * sum_j |x_j| / 32 + 1e-7 per element
(ten FP32 butterfly stages). A result rounded to bf16 may add half a bf16 ulp
of the value actually returned (bf16 keeps 8 significant bits, so that is
2^(floor(log2 |y|) - 8), between 2^-9 |y| and 2^-8 |y|).
"""
import functools

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


def bf16_half_ulp(y):
    """Half an ulp of bf16 at each returned value: the most round-to-nearest
    can move a value onto it (8 significant bits; zero for zero)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    out = np.zeros_like(a)
    nz = a > 0
    out[nz] = np.exp2(np.floor(np.log2(a[nz])) - 8.0)
    return out


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
    got = f64(out)
    if out_dtype == bt.BF16:
        tol = tol + bf16_half_ulp(got)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) / tol))


def test_fwht_matrix_form_small():
    xb = workloads.fwht_input(3, 2, 1024)
    s = workloads.sign1024()
    got = f64(bt.fwht1024(T(xb, "bf16"), T(s), bt.F32))
    ref = oracle.rotate(oracle.bf16_to_f64(xb), s, "matrix")
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


# ---------------------------------------------------------------- GEMV ----

def run_gemv(case, layout=bt.LAYOUT_B3, rotate=True, y_dtype=bt.F32, x_f32=None, checked=True):
    """bt_gemv on a case. checked=False passes no error word, which selects the
    kernels the benchmark times (code validation compiled out)."""
    codes = bt.pack(T(case["trits"]), layout)
    if rotate:
        x = T(case["x"], "bf16")
        sign = T(case["sign"])
    else:
        x = torch.from_numpy(x_f32.astype(np.float32)).to(DEV)
        sign = None
    err = torch.zeros(1, dtype=torch.int32, device=DEV) if checked else None
    y = bt.gemv(codes, T(case["scales"]), x, sign, case["N"], layout, y_dtype, dev_err=err)
    torch.cuda.synchronize()
    if checked:
        assert int(err.item()) == 0
    return f64(y)


def check(y, y_ref, bound, extra=0.0):
    r = np.abs(y - y_ref) / (bound + extra)
    assert np.all(r <= 1.0), f"max err/bound {float(r.max()):.4g}"
    print(f"max err/bound {float(r.max()):.4g}")
    return float(r.max())


def check_bf16(y, y_ref, bound):
    """The FP32 bound plus the bf16 rounding of the value actually returned."""
    return check(y, y_ref, bound, extra=bf16_half_ulp(y))


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_tiny_config(layout):
    case = workloads.layer_inputs("C0", workloads.TINY)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout), y_ref, b)


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemv_decode_triple_full_size(idx, layer, checked):
    case = workloads.layer_inputs("C1", layer, index=idx)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, checked=checked), y_ref, b)


# The 27B-equivalent sweep runs the triple's shapes at M = 1, 4 and 16. Every
# output element of the M = 4 and M = 16 calls is compared with the oracle, in
# both layouts, with the kernels the sweep times (no error word).
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M", [4, 16])
@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemv_sweep_shapes_full(layout, M, idx, layer):
    case = workloads.layer_inputs("C2", layer, M=M, index=idx)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout, checked=False), y_ref, b)


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


# Single-row (M = 1) calls with K % 1024 == 0 take the persistent
# table-lookup kernel: every CTA streams an equal contiguous share of the
# (chunk, row) items, one or several chunks. These cases cover its branches.

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
    # 76 blocks = 152 chunks of 512: more chunks than SMs, so CTAs cover several chunks
    N, K = 40, 76 * 1024
    case = workloads.random_case(2700, 1, N, K)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    check(run_gemv(case, layout), y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemv_m1_bf16_output(layout):
    case = workloads.random_case(2800, 1, 5120, 5120)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemv(case, layout, y_dtype=bt.BF16)
    check_bf16(y, y_ref, b)


def test_gemv_bf16_output():
    case = workloads.random_case(4000, 4, 512, 2048)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemv(case, y_dtype=bt.BF16)
    check_bf16(y, y_ref, b)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("t", [1, -1])
@pytest.mark.parametrize("K", [2048, 28 * 1024])
def test_gemv_special_cases_m1_exact(layout, t, K):
    # M = 1 runs the table-lookup kernel. A byte of zero trits has the table
    # entry 0 exactly and a byte with one non-zero trit the entry +-x'_k
    # exactly; every other term of the row, and every other chunk partial, is
    # an exact zero, so all-zero weights give y = 0 exactly and a single trit
    # gives y[n] = t * fl(s * x'_k), with x' the library's own FP32 rotation
    # (bt_fwht1024 runs the same warp transform).
    N = 64
    case = workloads.random_case(5000, 1, N, K)
    case["trits"] = np.zeros_like(case["trits"])
    for checked in (True, False):
        assert np.all(run_gemv(case, layout, checked=checked) == 0.0)
    n, k = 17, K - 548
    case["trits"][n, k] = t
    xr = bt.fwht1024(T(case["x"], "bf16"), T(case["sign"]), bt.F32).cpu().numpy()
    s = np.float32(case["scales"][n, k // 128].view(np.float16))
    expect = np.zeros(N, dtype=np.float32)
    expect[n] = np.float32(t) * (s * xr[0, k])
    assert abs(float(expect[n])) >= 2.0 ** -13
    for checked in (True, False):
        y1 = run_gemv(case, layout, checked=checked)[0].astype(np.float32)
        assert np.array_equal(y1, expect), (y1[n], expect[n])


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M,K", [(2, 2048), (4, 2048), (16, 2048), (3, 1152)])
def test_gemv_special_cases_batched(layout, M, K):
    # M > 1 runs the tensor-core path. Weights enter as digits t + 1; the
    # per-group correction is the same tensor-core sum taken with every digit
    # 1, so a row of zero trits cancels exactly: y = 0 bit for bit. (K = 1152:
    # pre-rotated input, the register-fed kernel.) A single trit stays within
    # the bound.
    N = 64
    case = workloads.random_case(5100 + M, M, N, K)
    case["trits"] = np.zeros_like(case["trits"])
    rotate = K % 1024 == 0
    xr = workloads.rng(5200 + M).standard_normal((M, K)).astype(np.float32).astype(np.float64)
    for checked in (True, False):
        y0 = run_gemv(case, layout, rotate=rotate, x_f32=None if rotate else xr, checked=checked)
        assert np.all(y0 == 0.0), float(np.max(np.abs(y0)))
    case["trits"][17, 1000] = -1
    if rotate:
        _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    else:
        y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check(run_gemv(case, layout, rotate=rotate, x_f32=None if rotate else xr), y_ref, b)


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

def run_gemm(trits, scales, x_bits, sign, layout=bt.LAYOUT_B3, x_f32=None, checked=True):
    codes = bt.pack(T(trits), layout)
    if x_f32 is None:
        x = T(x_bits, "bf16")
        sg = T(sign)
    else:
        x = torch.from_numpy(x_f32.astype(np.float32)).to(DEV)
        sg = None
    err = torch.zeros(1, dtype=torch.int32, device=DEV) if checked else None
    y = bt.gemm(codes, T(scales), x, sg, trits.shape[0], layout, dev_err=err)
    torch.cuda.synchronize()
    if checked:
        assert int(err.item()) == 0
    return f64(y)


def tile_rows(M, seed, per_tile=3):
    """Sampled rows of a prefill output: the first and last row of every
    128-row tile (so both CTAs of every 256-row pair) plus seeded rows inside."""
    g = workloads.rng(seed)
    rows = []
    for t0 in range(0, M, 128):
        rows += [t0, t0 + 127]
        rows += list(t0 + 1 + g.choice(126, size=per_tile - 2, replace=False))
    return np.array(sorted(set(rows)))


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
@pytest.mark.parametrize("M,N,K", [(128, 256, 1024), (256, 384, 2048), (128, 128, 3072)])
def test_gemm_small_full(layout, M, N, K):
    case = workloads.random_case(8000 + N + K, M, N, K)
    _, y_ref, b = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], layout)
    check_bf16(y, y_ref, b)


@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemm_prefill_triple_sampled_rows(idx, layer):
    # the pp512 shapes at full N and K, in the configuration the benchmark times
    # (no error word); the oracle computes whole rows of Y: three in every
    # 128-row tile, including each tile's first and last row
    case = workloads.layer_inputs("C3", layer, index=idx)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], checked=False)
    rows = tile_rows(512, 9000 + idx)
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check_bf16(y[rows], y_ref, b)


@pytest.mark.parametrize("idx,layer", list(enumerate(workloads.TRIPLE)))
def test_gemm_2bit_prefill_triple_sampled_rows(idx, layer):
    # layout A/B: the 2-bit twin on every pp512 shape
    case = workloads.layer_inputs("C4", layer, M=512, index=idx)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], bt.LAYOUT_2BIT, checked=False)
    rows = tile_rows(512, 9100 + idx)
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check_bf16(y[rows], y_ref, b)


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
    check_bf16(y, y_ref, b)


@functools.lru_cache(maxsize=2)
def _two_tile_case(N, K):
    # at M = 512, N = 17408 takes 256-wide weight tiles with two 256-row
    # activation tiles per CTA pair; N = 5120 takes 160-wide tiles with two
    # activation tiles per pair and K split in two (17 K groups: halves of 8
    # and 9), the two pairs of a tile sharing a cluster and swapping halves in
    # shared memory. Small K keeps the whole output cheap for the oracle; both
    # have odd numbers of K groups.
    M = 512
    case = workloads.random_case(8550 + N, M, N, K)
    xr = workloads.rng(8551 + N).standard_normal((M, K)) * 2.0
    xr32 = xr.astype(np.float32).astype(np.float64)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr32)
    return case, xr32, y_ref, b


@pytest.mark.parametrize("N,K", [(17408, 1152), (5120, 2176)])
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemm_two_tiles_per_pair_full(layout, N, K):
    case, xr32, y_ref, b = _two_tile_case(N, K)
    y = run_gemm(case["trits"], case["scales"], None, None, layout, x_f32=xr32)
    check_bf16(y, y_ref, b)
    # the splits meet whatever their timing: same bits each call
    y2 = run_gemm(case["trits"], case["scales"], None, None, layout, x_f32=xr32)
    assert np.array_equal(y, y2)


@pytest.mark.parametrize("M,K", [(128, 4096), (256, 2176)])
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemm_small_m_split_k_full(layout, M, K):
    # M = 128 and 256 against N = 5120 split K over the single-CTA kernel:
    # 32 K groups in four (8 each), 17 in two (8 and 9)
    N = 5120
    case = workloads.random_case(8570 + M, M, N, K)
    xr = workloads.rng(8571 + M).standard_normal((M, K)) * 2.0
    xr32 = xr.astype(np.float32).astype(np.float64)
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr32)
    y = run_gemm(case["trits"], case["scales"], None, None, layout, x_f32=xr32)
    check_bf16(y, y_ref, b)
    y2 = run_gemm(case["trits"], case["scales"], None, None, layout, x_f32=xr32)
    assert np.array_equal(y, y2)


@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemm_split_clusters_two_pairs_along_m_sampled_rows(layout):
    # M = 1024 against N = 5120: two clusters along M, each of two pairs with
    # two activation tiles and one half of K (24 K groups, rotated input)
    M, N, K = 1024, 5120, 3072
    case = workloads.random_case(8580 + layout, M, N, K)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"], layout)
    rows = tile_rows(M, 8581)
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check_bf16(y[rows], y_ref, b)


def test_gemm_two_tiles_per_pair_two_pairs_sampled_rows():
    # M = 1024: two pairs along M, each with two activation tiles
    M, N, K = 1024, 17408, 2048
    case = workloads.random_case(8560, M, N, K)
    y = run_gemm(case["trits"], case["scales"], case["x"], case["sign"])
    rows = tile_rows(M, 8561)
    xr = oracle.rotate_bf16(case["x"][rows], case["sign"])
    y_ref, b = oracle.gemv(case["trits"], case["scales"], xr)
    check_bf16(y[rows], y_ref, b)


@pytest.mark.parametrize("M", [128, 512])   # 512: the split-K pair kernel at N = 5120
@pytest.mark.parametrize("layout", [bt.LAYOUT_B3, bt.LAYOUT_2BIT])
def test_gemm_flags_invalid_codes(layout, M):
    N, K = (128, 1024) if M == 128 else (5120, 2048)
    case = workloads.random_case(8650 + M, M, N, K)
    codes = oracle.pack(case["trits"], layout)
    codes[N - 3, 40] = 247 if layout == bt.LAYOUT_B3 else 0xC3
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = bt.gemm(T(codes), T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), N, layout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bt.DEVERR_INVALID_CODE
    assert torch.isfinite(y.float()).all()
    # and a clean call on the same shape reports nothing
    err.zero_()
    bt.gemm(T(oracle.pack(case["trits"], layout)), T(case["scales"]), T(case["x"], "bf16"), T(case["sign"]), N,
            layout, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


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
    check_bf16(y1, y_ref, b)


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
