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


def _digits_by_divmod(code):
    # base-3 digits of a byte, least significant first, by repeated division
    out = []
    for _ in range(5):
        code, d = divmod(code, 3)
        out.append(d)
    return out


@pytest.mark.parametrize("K", [128, 640, 1024, 5120, 17408])
def test_pack_continuous_layout(K):
    # byte j holds trits 5j .. 5j+4 of the row across group boundaries; read
    # back here by plain division, independently of the oracle's unpack
    g = workloads.rng(9 + K)
    t = workloads.trits(g, 3, K)
    codes = oracle.pack(t, oracle.LAYOUT_BASE3_CONT)
    used = -(-K // 5)
    assert codes.shape == (3, -(-used // 16) * 16)
    for n in range(3):
        flat = []
        for j in range(used):
            flat += [d - 1 for d in _digits_by_divmod(int(codes[n, j]))]
        assert flat[:K] == t[n].tolist()
        assert all(v == 0 for v in flat[K:])             # pad trits: digit 1
        assert not codes[n, used:].any()                # row padding: zero bytes
    assert np.array_equal(oracle.unpack(codes, K, oracle.LAYOUT_BASE3_CONT), t)


def test_pack_continuous_worked_example_and_bits():
    rows = dict((r[0], r[1:]) for r in _read_golden("pack_example.txt"))
    example = [int(v) for v in rows["trits"]]
    t = np.zeros((1, 5120), dtype=np.int8)
    t[0, :5] = example
    codes = oracle.pack(t, oracle.LAYOUT_BASE3_CONT)
    assert int(codes[0, 0]) == 183
    # the release summary's accounting: 1.6 bit per trit + 16 bit per 128 = 1.725 bit at K = 5120
    K = 5120
    bits = (oracle.row_bytes(oracle.LAYOUT_BASE3_CONT, K) * 8 + (K // 128) * 16) / K
    assert bits == 1.725
    assert (oracle.row_bytes(oracle.LAYOUT_BASE3, K) * 8 + (K // 128) * 16) / K == 1.75
    # a group boundary inside a byte: trits 125..129 share byte 25
    t2 = np.zeros((1, 256), dtype=np.int8)
    t2[0, 125:130] = [1, -1, 1, -1, 1]
    c2 = oracle.pack(t2, oracle.LAYOUT_BASE3_CONT)
    assert _digits_by_divmod(int(c2[0, 25])) == [2, 0, 2, 0, 2]


def test_pack_continuous_rejects_invalid():
    ok = oracle.pack(np.zeros((1, 128), dtype=np.int8), oracle.LAYOUT_BASE3_CONT)  # 26 bytes used of 32
    assert ok.shape == (1, 32)
    c = ok.copy()
    c[0, 4] = 243
    assert oracle.unpack_status(c, 128, oracle.LAYOUT_BASE3_CONT) == oracle.BAD_CODE
    c = ok.copy()
    c[0, 25] = 121 - 27                                   # a pad trit of the last byte that is not 0
    assert oracle.unpack_status(c, 128, oracle.LAYOUT_BASE3_CONT) == oracle.BAD_PAD
    c = ok.copy()
    c[0, 30] = 1                                          # row padding must be zero
    assert oracle.unpack_status(c, 128, oracle.LAYOUT_BASE3_CONT) == oracle.BAD_PAD


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


# ------------------------------------------------ offline ternarisation ----

def test_double_to_f16_matches_numpy_round_to_nearest_even():
    g = np.random.default_rng(7)
    v = g.standard_normal(100000) * np.exp2(g.integers(-30, 17, 100000))
    edge = [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14,
            -0.999 * 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0]
    v = np.concatenate([v, edge])
    ours = np.array([oracle.double_to_f16(x) for x in v], dtype=np.uint16)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def _rotated_basis_weights(v_rot, sign):
    """Float W whose block-wise rotation R W^T is exactly v_rot: W = S . (H v) / 32
    with scipy's Hadamard (R^T = S H / 32, H symmetric); exact for these values."""
    import scipy.linalg
    H = scipy.linalg.hadamard(1024).astype(np.float64)
    N, K = v_rot.shape
    W = np.zeros_like(v_rot)
    for b in range(K // 1024):
        blk = v_rot[:, 1024 * b:1024 * (b + 1)]
        W[:, 1024 * b:1024 * (b + 1)] = (blk @ H.T) / 32.0 * sign[None, :].astype(np.float64)
    return W


def test_ternarize_recovers_a_ternary_target_exactly():
    # rotated rows that are exactly c * t: the ternariser must return t and c
    g = np.random.default_rng(11)
    N, K = 6, 2048
    sign = workloads.sign1024()
    t = g.choice([-1, 0, 1], size=(N, K), p=[0.3, 0.4, 0.3]).astype(np.int8)
    t[2, 128:256] = 0                                   # one all-zero group: scale 0
    c = 2.0 ** -3
    W = _rotated_basis_weights(c * t.astype(np.float64), sign)
    assert np.array_equal(oracle.rotate(W, sign), c * t)   # the construction is exact
    trits, scales = oracle.ternarize(W, sign)
    assert np.array_equal(trits, t)
    expect = np.full((N, K // 128), np.float16(c).view(np.uint16), dtype=np.uint16)
    expect[2, 1] = 0
    assert np.array_equal(scales, expect)


def test_ternarize_sign_and_power_of_two_equivariance():
    g = np.random.default_rng(12)
    W = g.standard_normal((5, 1024)) * 0.05
    sign = workloads.sign1024()
    t, s = oracle.ternarize(W, sign)
    tn, sn = oracle.ternarize(-W, sign)
    assert np.array_equal(tn, -t) and np.array_equal(sn, s)
    t4, s4 = oracle.ternarize(W * 4.0, sign)
    assert np.array_equal(t4, t)
    assert np.array_equal(oracle.f16_to_f64(s4), 4.0 * oracle.f16_to_f64(s))


def _group_errors(v, t, s_bits):
    s = oracle.f16_to_f64(s_bits)
    rec = t.reshape(v.shape[0], -1, 128) * s[:, :, None]
    return ((v.reshape(v.shape[0], -1, 128) - rec) ** 2).sum(axis=2)


def test_ternarize_is_no_worse_than_the_half_mean_threshold():
    # the search includes tau = 0.5 mean|v| (the pages' fixed +-0.5-style rule),
    # so its error is never above that rule's error, computed here on its own
    g = np.random.default_rng(13)
    W = g.standard_normal((8, 2048)) * 0.02
    W.reshape(-1)[g.choice(W.size, 40, replace=False)] *= 25.0
    sign = workloads.sign1024()
    t, s = oracle.ternarize(W, sign)
    v = oracle.rotate(W, sign)
    vg = v.reshape(8, -1, 128)
    tau = 0.5 * np.abs(vg).mean(axis=2, keepdims=True)
    keep = np.abs(vg) >= tau
    s_half = np.array([[np.float16((np.abs(vg[n, q])[keep[n, q]]).mean()).view(np.uint16)
                        for q in range(vg.shape[1])] for n in range(8)], dtype=np.uint16)
    t_half = (np.sign(vg) * keep).astype(np.int8).reshape(8, 2048)
    assert np.all(_group_errors(v, t, s) <= _group_errors(v, t_half, s_half) + 1e-18)


def test_rotation_lowers_the_ternarisation_error_on_outlier_weights():
    # the pages' reason for R: spreading outliers before ternarising. Rotated
    # ternarisation error (in the rotated basis, equal to the error in the
    # original one since R is orthogonal) against ternarising W as it is (fed
    # as R^T W, which the ternariser rotates back to W).
    g = np.random.default_rng(14)
    N, K = 16, 2048
    W = g.standard_normal((N, K)) * 0.02
    W.reshape(-1)[g.choice(W.size, W.size // 100, replace=False)] *= 20.0
    sign = workloads.sign1024()
    t, s = oracle.ternarize(W, sign)
    err_rot = _group_errors(oracle.rotate(W, sign), t, s).sum()
    Wt = _rotated_basis_weights(W, sign)            # R^T W
    t0, s0 = oracle.ternarize(Wt, sign)
    err_plain = _group_errors(oracle.rotate(Wt, sign), t0, s0).sum()
    assert err_rot < 0.8 * err_plain, (err_rot, err_plain)
