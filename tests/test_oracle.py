"""Pins for the CPU oracle (no GPU).

Each test ties an oracle routine to something other than the oracle itself:
the pages' worked example and printed matrix (tests/golden), exhaustive
enumeration, scipy / numpy library routines, closed forms and invariants.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- packing ----

def test_pack_worked_example_183():
    rows = dict((r[0], r[1:]) for r in _read_golden("pack_example.txt"))
    example = [int(v) for v in rows["trits"]]
    expected = int(rows["code"][0])
    t = np.zeros((1, 128), dtype=np.int8)
    t[0, :5] = example
    codes = oracle.pack(t)
    assert codes.shape == (1, 26)
    assert int(codes[0, 0]) == expected == 183
    assert oracle.unpack(codes, 128)[0, :5].tolist() == example


def test_pack_base3_exhaustive_243():
    # every 5-trit tuple lands in a distinct byte 0..242 equal to the base-3 number
    tuples = list(itertools.product((-1, 0, 1), repeat=5))
    t = np.zeros((len(tuples), 128), dtype=np.int8)
    for r, tup in enumerate(tuples):
        t[r, :5] = tup
    codes = oracle.pack(t)
    first = codes[:, 0].astype(int)
    assert sorted(first.tolist()) == list(range(243))
    for r, tup in enumerate(tuples):
        assert first[r] == sum((v + 1) * 3 ** i for i, v in enumerate(tup))
    assert np.array_equal(oracle.unpack(codes, 128), t)


def test_pack_2bit_exhaustive_81():
    tuples = list(itertools.product((-1, 0, 1), repeat=4))
    t = np.zeros((len(tuples), 128), dtype=np.int8)
    for r, tup in enumerate(tuples):
        t[r, :4] = tup
    codes = oracle.pack(t, oracle.LAYOUT_2BIT)
    assert codes.shape == (81, 32)
    for r, tup in enumerate(tuples):
        assert int(codes[r, 0]) == sum((v + 1) << (2 * i) for i, v in enumerate(tup))
    assert np.array_equal(oracle.unpack(codes, 128, oracle.LAYOUT_2BIT), t)


def test_pack_group_layout_and_padding():
    g = workloads.rng(7)
    t = workloads.trits(g, 5, 384)
    codes = oracle.pack(t)
    assert codes.shape == (5, 3 * 26)
    c3 = codes.reshape(5, 3, 26).astype(int)
    # byte b of group j holds trits 128 j + 5 b + i, i = 0..4, digit (t + 1) * 3^i
    for n in range(5):
        for j in range(3):
            for b in range(25):
                want = sum((int(t[n, 128 * j + 5 * b + i]) + 1) * 3 ** i for i in range(5))
                assert c3[n, j, b] == want
            last = sum((int(t[n, 128 * j + 125 + i]) + 1) * 3 ** i for i in range(3)) + 27 + 81
            assert c3[n, j, 25] == last
    assert c3[:, :, 25].min() >= 108 and c3[:, :, 25].max() <= 134
    assert np.array_equal(oracle.unpack(codes, 384), t)


def test_pack_2bit_layout_random_roundtrip():
    g = workloads.rng(8)
    t = workloads.trits(g, 7, 256)
    codes = oracle.pack(t, oracle.LAYOUT_2BIT)
    c = codes.astype(int)
    for n in range(7):
        for k in range(256):
            assert (c[n, k // 4] >> (2 * (k % 4))) & 3 == int(t[n, k]) + 1
    assert np.array_equal(oracle.unpack(codes, 256, oracle.LAYOUT_2BIT), t)


def test_pack_rejects_invalid():
    t = np.zeros((1, 128), dtype=np.int8)
    t[0, 17] = 2
    with pytest.raises(oracle.OracleError):
        oracle.pack(t)
    ok = oracle.pack(np.zeros((1, 128), dtype=np.int8))
    for bad in range(243, 256):
        c = ok.copy()
        c[0, 3] = bad
        assert oracle.unpack_status(c, 128) == oracle.BAD_CODE
    c = ok.copy()
    c[0, 25] = 121 - 27  # pad digit 3 -> 0
    assert oracle.unpack_status(c, 128) == oracle.BAD_PAD
    c2 = oracle.pack(np.zeros((1, 128), dtype=np.int8), oracle.LAYOUT_2BIT)
    c2[0, 5] = 0xFF
    assert oracle.unpack_status(c2, 128, oracle.LAYOUT_2BIT) == oracle.BAD_CODE
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.zeros((1, 100), dtype=np.int8))


# ------------------------------------------------------ number formats -----

def test_f16_conversion_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_conversion_samples():
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(ours[~nan], ref[~nan])


# ----------------------------------------------------------- Hadamard -------

def test_hadamard_h4_printed():
    H4 = np.array([[int(v) for v in r] for r in _read_golden("hadamard4.txt")], dtype=np.int8)
    assert np.array_equal(oracle.hadamard(4), H4)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
def test_hadamard_matches_scipy_and_is_orthogonal(n):
    H = oracle.hadamard(n)
    assert np.array_equal(H, scipy.linalg.hadamard(n).astype(np.int8))
    Hd = H.astype(np.int64)
    assert np.array_equal(Hd @ Hd.T, n * np.eye(n, dtype=np.int64))


# ----------------------------------------------------------- rotation -------

def test_rotation_matrix_equals_butterfly():
    x = workloads.rng(11).standard_normal((3, 2048))
    s = workloads.sign1024()
    a = oracle.rotate(x, s, "matrix")
    b = oracle.rotate(x, s, "butterfly")
    assert np.max(np.abs(a - b)) < 1e-12 * np.max(np.abs(a))


def test_rotation_is_orthogonal():
    s = workloads.sign1024()
    R_rows = oracle.rotate(np.eye(1024), s, "matrix")      # row j = R e_j
    assert np.max(np.abs(R_rows @ R_rows.T - np.eye(1024))) < 1e-12
    # R e_j = s_j H[:, j] / 32
    H = scipy.linalg.hadamard(1024).astype(np.float64)
    assert np.max(np.abs(R_rows - (s[:, None] * H.T) / 32.0)) < 1e-15


def test_rotation_closed_forms():
    s = workloads.sign1024().astype(np.float64)
    # R (S . 1) = H 1 / 32 = 32 e_0, independently in each block
    x = np.tile(s, 3)[None, :]
    r = oracle.rotate(x, s.astype(np.int8), "butterfly")
    expect = np.zeros(3 * 1024)
    expect[[0, 1024, 2048]] = 32.0
    assert np.array_equal(r[0], expect)
    # Parseval per block and blockwise independence
    g = workloads.rng(12)
    x = g.standard_normal((2, 4096))
    r = oracle.rotate(x, s.astype(np.int8), "butterfly")
    for b in range(4):
        sl = slice(1024 * b, 1024 * (b + 1))
        assert abs(np.sum(r[:, sl] ** 2) - np.sum(x[:, sl] ** 2)) < 1e-9 * np.sum(x[:, sl] ** 2)
    y = x.copy()
    y[:, 1024:2048] = 0
    r2 = oracle.rotate(y, s.astype(np.int8), "butterfly")
    assert np.array_equal(r2[:, :1024], r[:, :1024]) and np.all(r2[:, 1024:2048] == 0)


def test_rotation_sign_applied_before_hadamard():
    # x = e_j: S is applied first, so R e_j = s_j * (column j of H) / 32
    s = workloads.sign1024()
    j = int(np.nonzero(s < 0)[0][3])
    x = np.zeros((1, 1024))
    x[0, j] = 1.0
    r = oracle.rotate(x, s, "matrix")[0]
    H = scipy.linalg.hadamard(1024)
    assert np.array_equal(r, -H[:, j] / 32.0)


# ---------------------------------------------------------- product --------

def test_dequant_matches_numpy():
    g = workloads.rng(13)
    t = workloads.trits(g, 9, 256)
    sc = workloads.scales_f16_bits(g, 9, 256)
    W = oracle.dequant(t, sc)
    ref = np.repeat(sc.view(np.float16).astype(np.float64), 128, axis=1) * t
    assert np.array_equal(W, ref)


def test_gemv_matches_numpy_matmul_on_dequantised_w():
    case = workloads.random_case(21, M=3, N=256, K=1024)
    xr = oracle.rotate_bf16(case["x"], case["sign"])
    y, bound = oracle.gemv(case["trits"], case["scales"], xr)
    W = np.repeat(case["scales"].view(np.float16).astype(np.float64), 128, axis=1) * case["trits"]
    ref = xr @ W.T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    mag = np.abs(xr) @ np.abs(W).T
    assert np.allclose(bound, 2e-3 * mag + 1e-5, rtol=1e-12, atol=0)


def test_gemv_brute_force_tiny():
    for seed, (M, N, K) in enumerate([(1, 1, 128), (2, 3, 256), (4, 8, 1024)]):
        case = workloads.random_case(100 + seed, M, N, K)
        xr = workloads.rng(200 + seed).standard_normal((M, K))
        y, _ = oracle.gemv(case["trits"], case["scales"], xr)
        sc = case["scales"].view(np.float16)
        for m in range(M):
            for n in range(N):
                acc = 0.0
                for k in range(K):
                    acc += float(sc[n, k // 128]) * int(case["trits"][n, k]) * xr[m, k]
                assert abs(acc - y[m, n]) <= 1e-12 * max(1.0, abs(acc))


def test_gemv_special_cases():
    case = workloads.random_case(31, 2, 16, 1024)
    xr = oracle.rotate_bf16(case["x"], case["sign"])
    y0, b0 = oracle.gemv(np.zeros_like(case["trits"]), case["scales"], xr)
    assert np.all(y0 == 0) and np.all(b0 == 1e-5)
    t = np.zeros_like(case["trits"])
    t[5, 700] = -1
    y1, _ = oracle.gemv(t, case["scales"], xr)
    s = float(case["scales"].view(np.float16)[5, 700 // 128])
    assert np.array_equal(y1[:, 5], -s * xr[:, 700])
    assert np.all(y1[:, np.arange(16) != 5] == 0)


def test_forward_is_gemv_of_rotation():
    case = workloads.random_case(41, 1, 32, 2048)
    xr, y, _ = oracle.forward(case["trits"], case["scales"], case["x"], case["sign"])
    x = (case["x"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s = case["sign"].astype(np.float64)
    H = scipy.linalg.hadamard(1024).astype(np.float64)
    ref_xr = np.concatenate([(H @ (s * x[0, b * 1024:(b + 1) * 1024])) / 32.0 for b in range(2)])
    assert np.max(np.abs(xr[0] - ref_xr)) < 1e-12 * np.max(np.abs(ref_xr))
