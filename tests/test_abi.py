"""The C ABI on the host: libbt.so loads, exports every entry point that
include/bt.h declares, and rejects bad arguments before launching anything.
No GPU is needed: every call below fails host-side validation."""
import ctypes
import os
import re

import pytest

import oracle
import ternary_weight_fwht1024_b200 as bt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return bt.load()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "bt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bt_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert _declared_functions() == sorted(bt.SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert lib.bt_version() >= 1
    assert bt.status_string(0) == "ok"
    for s in range(1, 7):
        assert bt.status_string(s) != "unknown status"
    assert bt.status_string(99) == "unknown status"


def test_codes_row_bytes(lib):
    assert bt.codes_row_bytes(bt.LAYOUT_B3, 1024) == 208
    assert bt.codes_row_bytes(bt.LAYOUT_B3, 5120) == 1040
    assert bt.codes_row_bytes(bt.LAYOUT_B3, 17408) == 3536
    assert bt.codes_row_bytes(bt.LAYOUT_2BIT, 5120) == 1280
    assert bt.codes_row_bytes(bt.LAYOUT_B3, 100) == -1
    assert bt.codes_row_bytes(bt.LAYOUT_B3, 0) == -1
    assert bt.codes_row_bytes(5, 1024) == -1
    # continuous base-3: ceil(K/5) bytes rounded up to 16, as the oracle lays them out
    for K in (128, 640, 1024, 5120, 17408):
        assert bt.codes_row_bytes(bt.LAYOUT_B3C, K) == oracle.row_bytes(oracle.LAYOUT_BASE3_CONT, K)
    assert bt.codes_row_bytes(bt.LAYOUT_B3C, 5120) == 1024 and bt.codes_row_bytes(bt.LAYOUT_B3C, 17408) == 3488


P = ctypes.c_void_p


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_pack_validation(lib):
    good = _fake(1 << 20)
    assert lib.bt_pack(7, good, 4, 128, good, None, None) == 1          # bad layout
    assert lib.bt_pack(0, good, 4, 100, good, None, None) == 2          # K % 128
    assert lib.bt_pack(0, good, -1, 128, good, None, None) == 2         # N < 0
    assert lib.bt_pack(0, None, 4, 128, good, None, None) == 1          # NULL
    assert lib.bt_pack(0, _fake((1 << 20) + 1), 4, 128, good, None, None) == 3  # align
    assert lib.bt_pack(0, None, 0, 128, None, None, None) == 0          # empty: no-op


def test_fwht_validation(lib):
    good = _fake(1 << 20)
    assert lib.bt_fwht1024(good, good, 1, 1000, 0, good, None) == 2
    assert lib.bt_fwht1024(good, good, 1, 1024, 5, good, None) == 1
    assert lib.bt_fwht1024(None, good, 1, 1024, 0, good, None) == 1
    assert lib.bt_fwht1024(_fake((1 << 20) + 8), good, 1, 1024, 0, good, None) == 3
    assert lib.bt_fwht1024(good, good, 0, 1024, 0, good, None) == 0


def test_gemv_validation(lib):
    g = _fake(1 << 20)
    args = lambda **kw: [kw.get("layout", 0), g, g, g, kw.get("xd", 1), kw.get("sign", g),
                         kw.get("M", 1), kw.get("N", 256), kw.get("K", 1024), kw.get("yd", 0),
                         kw.get("y", g), kw.get("ws", None), kw.get("wsb", 0), None, None]
    assert lib.bt_gemv(*args(layout=3)) == 1
    assert lib.bt_gemv(*args(M=17)) == 2
    assert lib.bt_gemv(*args(K=1000)) == 2
    assert lib.bt_gemv(*args(K=1152)) == 2            # rotation needs K % 1024
    assert lib.bt_gemv(*args(xd=0)) == 1              # raw activations must be bf16
    assert lib.bt_gemv(*args(yd=4)) == 1
    assert lib.bt_gemv(*args(y=None)) == 1
    assert lib.bt_gemv(*args(y=_fake((1 << 20) + 4))) == 3
    assert lib.bt_gemv(*args()) == 4                  # no workspace
    need = lib.bt_gemv_workspace_bytes(0, 1, 256, 1024)
    assert need > 0
    assert lib.bt_gemv(*args(ws=_fake(1 << 24), wsb=need - 1)) == 4
    assert lib.bt_gemv(*args(ws=_fake((1 << 24) + 16), wsb=need)) == 3
    assert lib.bt_gemv(*args(M=0)) == 0
    assert lib.bt_gemv_workspace_bytes(0, 17, 256, 1024) == 0
    # continuous base-3: single rows only, K % 1024 == 0, 16-byte aligned codes and scales
    assert lib.bt_gemv(*args(layout=2, M=2)) == 2
    assert lib.bt_gemv(*args(layout=2, K=1152, sign=None)) == 2
    assert lib.bt_gemv(*args(layout=2)) == 4          # fine, but no workspace
    assert lib.bt_gemv_workspace_bytes(2, 2, 256, 1024) == 0
    assert lib.bt_gemv_workspace_bytes(2, 1, 256, 1024) == 256 * 2 * 4  # two 640-column chunks of partials


def test_gemm_validation(lib):
    g = _fake(1 << 20)
    args = lambda **kw: [kw.get("layout", 0), g, g, g, 1, g, kw.get("M", 512), kw.get("N", 5120),
                         kw.get("K", 5120), g, kw.get("ws", None), kw.get("wsb", 0), None, None]
    assert lib.bt_gemm(*args(M=100)) == 2
    assert lib.bt_gemm(*args(N=1000)) == 2
    assert lib.bt_gemm(*args(K=1000)) == 2
    assert lib.bt_gemm(*args()) == 4
    assert lib.bt_gemm_workspace_bytes(0, 512, 5120, 5120) > 0
    assert lib.bt_gemm_workspace_bytes(0, 100, 5120, 5120) == 0
    assert lib.bt_gemm(*args(layout=2)) == 1           # the prefill GEMM reads group-aligned bytes only
    assert lib.bt_gemm_workspace_bytes(2, 512, 5120, 5120) == 0


def test_gemm_workspace_sizes(lib):
    # without a GPU the tile choice assumes B200's 148 SMs. The rotated FP16
    # activations and the row scales, each rounded up to 256 bytes ...
    def base(M, K):
        return -(-M * K * 2 // 256) * 256 + -(-M * 4 // 256) * 256
    # ... are all that 17408 x 5120 needs (256-wide tiles, two activation
    # tiles per pair, 136 CTAs)
    assert lib.bt_gemm_workspace_bytes(0, 512, 17408, 5120) == base(512, 5120)
    # N = 5120 at M = 512 splits K in two over 160-wide tiles; the two pairs
    # of a tile share a cluster and swap halves in shared memory: nothing more
    for K in (2176, 5120, 17408):
        for layout in (0, 1):
            assert lib.bt_gemm_workspace_bytes(layout, 512, 5120, K) == base(512, K)
    # 15 K groups are too few to split: 2-bit takes 80-wide tiles, base-3
    # 160-wide ones with one activation tile per pair
    for layout in (0, 1):
        assert lib.bt_gemm_workspace_bytes(layout, 512, 5120, 1920) == base(512, 1920)
    # M = 128 and 256 against N = 5120 fill the SMs by splitting K over the
    # single-CTA kernel with 160-wide tiles (20 decoder warps): 4 ways for
    # 32 tiles, 2 ways for 64
    assert lib.bt_gemm_workspace_bytes(0, 128, 5120, 5120) == base(128, 5120) + 32 * 20 * 4 + 4 * 128 * 5120 * 4
    assert lib.bt_gemm_workspace_bytes(0, 256, 5120, 5120) == base(256, 5120) + 64 * 20 * 4 + 2 * 256 * 5120 * 4
    # 24 K groups allow 3 splits at most
    assert lib.bt_gemm_workspace_bytes(1, 128, 5120, 3072) == base(128, 3072) + 32 * 20 * 4 + 3 * 128 * 5120 * 4
    # 17408 columns fill the SMs without a split
    assert lib.bt_gemm_workspace_bytes(0, 128, 17408, 5120) == base(128, 5120)


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        bt.pack(torch.zeros((2, 128), dtype=torch.int8))


def test_batched_validation(lib):
    good = 1 << 20

    def probs(**kw):
        arr = (bt.GemvProblem * 2)()
        for i in range(2):
            arr[i].codes = arr[i].scales = arr[i].x = arr[i].y = good
            arr[i].x_dtype, arr[i].x_from, arr[i].N, arr[i].K = 1, -1, 64, 1024
        for k, v in kw.items():
            setattr(arr[1], k, v)
        return arr
    call = lambda a, sign=None: lib.bt_gemv_batched(0, a, 2, sign, 0, None, 0, None, None)  # noqa: E731
    assert call(probs()) == 4                       # fine but no workspace
    assert call(probs(K=1000)) == 2                 # K % 1024
    assert call(probs(K=76 * 1024)) == 4            # any K % 1024 == 0
    assert call(probs(N=(1 << 24) + 1)) == 2         # rows beyond 2^24
    assert call(probs(x_from=1)) == 1               # only earlier outputs
    assert call(probs(x_from=0, K=1024, N=64)) == 2  # problem 0's N (64) is not this K
    assert call(probs(x_from=-2)) == 1
    assert call(probs(y=good + 8)) == 3             # alignment
    assert call(probs(x_dtype=0), _fake(good)) == 1  # rotation reads bf16
    assert lib.bt_gemv_batched(0, probs(), 0, None, 0, None, 0, None, None) == 0  # nothing to do
    arr = probs()
    need = lib.bt_gemv_batched_workspace_bytes(0, arr, 2)
    assert need == 256 * ((2 * 64 * 2 * 4 + 255) // 256)  # a float per (row, 512-chunk) of the group
    arr = probs(x_from=0, K=64 * 1024)
    arr[0].N = 64 * 1024                              # problem 1 reads problem 0: two groups
    need = lib.bt_gemv_batched_workspace_bytes(0, arr, 2)
    assert need == (64 * 1024 * 2 + 64 * 128) * 4       # every matrix keeps its partials until the end


def test_noalloc_limits_stated_in_the_header(lib):
    # the 8 MiB built-in scratch: the largest M that fits on each decode shape, as bt.h states it
    lim = 8 << 20
    for layout in (bt.LAYOUT_B3, bt.LAYOUT_2BIT):
        for (N, K), mmax in (((5120, 5120), 16), ((5120, 17408), 11), ((17408, 5120), 11), ((17408, 17408), 3)):
            assert lib.bt_gemv_workspace_bytes(layout, mmax, N, K) <= lim
            if mmax < 16:
                assert lib.bt_gemv_workspace_bytes(layout, mmax + 1, N, K) > lim
    assert lib.bt_gemv_workspace_bytes(0, 1, 32768, 32768) <= lim
    assert lib.bt_gemv_workspace_bytes(0, 1, 33792, 33792) > lim
