"""CPU oracle for the ternary-weight FWHT-1024 path -- TEST INFRASTRUCTURE.

Plain FP64 C (``bt_oracle.c``) behind ctypes, plus numpy glue. Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The CUDA library shares no code with it and never calls
it. What each routine follows is stated in ``bt_oracle.c``.

Every routine here is pinned by a ``-m "not gpu"`` test against something
other than itself: the pages' worked example (183) and printed H4, an
exhaustive pack/unpack round trip, scipy's Hadamard construction, the
orthogonality of R, closed forms, and numpy's float64 matmul on the
dequantised matrix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bt_oracle.c")
_LIB = os.path.join(_HERE, "libbt_oracle.so")
_lock = threading.Lock()
_lib = None

LAYOUT_BASE3 = 0
LAYOUT_2BIT = 1
LAYOUT_BASE3_CONT = 2
GROUP = 128
BLOCK = 1024

OK, BAD_SHAPE, BAD_TRIT, BAD_CODE, BAD_PAD, BAD_LAYOUT = range(6)


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile bt_oracle.c into libbt_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_bytes_per_group.argtypes = [ctypes.c_int]
            lib.oracle_row_bytes.argtypes = [ctypes.c_int, I64]
            lib.oracle_row_bytes.restype = I64
            lib.oracle_pack.argtypes = [ctypes.c_int, P, I64, I64, P]
            lib.oracle_unpack.argtypes = [ctypes.c_int, P, I64, I64, P]
            lib.oracle_hadamard.argtypes = [I64, P]
            lib.oracle_rotate_matrix.argtypes = [P, P, I64, I64, P]
            lib.oracle_rotate_butterfly.argtypes = [P, P, I64, I64, P]
            lib.oracle_dequant.argtypes = [P, P, I64, I64, P]
            lib.oracle_gemv.argtypes = [P, P, P, I64, I64, I64, P, P]
            lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_f16_array_to_double.argtypes = [P, I64, P]
            lib.oracle_bf16_array_to_double.argtypes = [P, I64, P]
            lib.oracle_double_to_f16.argtypes = [ctypes.c_double]
            lib.oracle_double_to_f16.restype = ctypes.c_uint16
            lib.oracle_ternarize.argtypes = [P, P, I64, I64, P, P]
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


def threads() -> int:
    return _load().oracle_threads()


def set_threads(n: int) -> None:
    """Host threads the oracle's parallel loops use from now on (timing only)."""
    _load().oracle_set_threads(int(n))


def bytes_per_group(layout: int) -> int:
    return _load().oracle_bytes_per_group(layout)


def row_bytes(layout: int, K: int) -> int:
    """Bytes of one packed row: K/128 groups of 26 (base-3) or 32 (2-bit), or
    ceil(K/5) rounded up to 16 (continuous base-3)."""
    return int(_load().oracle_row_bytes(layout, K))


def pack(trits: np.ndarray, layout: int = LAYOUT_BASE3) -> np.ndarray:
    t = np.ascontiguousarray(trits, dtype=np.int8)
    N, K = t.shape
    rb = row_bytes(layout, K)
    if rb < 0:
        _check(BAD_SHAPE, "pack")
    codes = np.zeros((N, rb), dtype=np.uint8)
    _check(_load().oracle_pack(layout, _ptr(t), N, K, _ptr(codes)), "pack")
    return codes


def unpack(codes: np.ndarray, K: int, layout: int = LAYOUT_BASE3) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    N = c.shape[0]
    t = np.zeros((N, K), dtype=np.int8)
    _check(_load().oracle_unpack(layout, _ptr(c), N, K, _ptr(t)), "unpack")
    return t


def unpack_status(codes: np.ndarray, K: int, layout: int = LAYOUT_BASE3) -> int:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    t = np.zeros((c.shape[0], K), dtype=np.int8)
    return _load().oracle_unpack(layout, _ptr(c), c.shape[0], K, _ptr(t))


def hadamard(n: int) -> np.ndarray:
    H = np.zeros((n, n), dtype=np.int8)
    _check(_load().oracle_hadamard(n, _ptr(H)), "hadamard")
    return H


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.zeros(b.shape, dtype=np.float64)
    _load().oracle_f16_array_to_double(_ptr(b), b.size, _ptr(out))
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.zeros(b.shape, dtype=np.float64)
    _load().oracle_bf16_array_to_double(_ptr(b), b.size, _ptr(out))
    return out


def rotate(x: np.ndarray, sign: np.ndarray, method: str = "butterfly") -> np.ndarray:
    """x' = (1/32) H_1024 (S . x) per 1024-block of each row. x: float64 [M, K]."""
    xx = np.ascontiguousarray(x, dtype=np.float64)
    s = np.ascontiguousarray(sign, dtype=np.int8)
    M, K = xx.shape
    out = np.zeros_like(xx)
    fn = _load().oracle_rotate_matrix if method == "matrix" else _load().oracle_rotate_butterfly
    _check(fn(_ptr(xx), _ptr(s), M, K, _ptr(out)), "rotate")
    return out


def rotate_bf16(x_bits: np.ndarray, sign: np.ndarray, method: str = "butterfly") -> np.ndarray:
    return rotate(bf16_to_f64(x_bits), sign, method)


def dequant(trits: np.ndarray, scales_bits: np.ndarray) -> np.ndarray:
    t = np.ascontiguousarray(trits, dtype=np.int8)
    s = np.ascontiguousarray(scales_bits, dtype=np.uint16)
    N, K = t.shape
    W = np.zeros((N, K), dtype=np.float64)
    _check(_load().oracle_dequant(_ptr(t), _ptr(s), N, K, _ptr(W)), "dequant")
    return W


def gemv(trits: np.ndarray, scales_bits: np.ndarray, xr: np.ndarray):
    """(y, bound), both float64 [M, N]: y = x' W^T with W = s * t (g128)."""
    t = np.ascontiguousarray(trits, dtype=np.int8)
    s = np.ascontiguousarray(scales_bits, dtype=np.uint16)
    x = np.ascontiguousarray(xr, dtype=np.float64)
    N, K = t.shape
    M = x.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    b = np.zeros((M, N), dtype=np.float64)
    _check(_load().oracle_gemv(_ptr(t), _ptr(s), _ptr(x), M, N, K, _ptr(y), _ptr(b)), "gemv")
    return y, b


def forward(trits: np.ndarray, scales_bits: np.ndarray, x_bits: np.ndarray, sign: np.ndarray):
    """The whole path y = W (R x) from bf16 activations: (x', y, bound)."""
    xr = rotate_bf16(x_bits, sign)
    y, b = gemv(trits, scales_bits, xr)
    return xr, y, b


def double_to_f16(v: float) -> int:
    """FP16 bit pattern of v, round to nearest even."""
    return int(_load().oracle_double_to_f16(float(v)))


def ternarize(W: np.ndarray, sign: np.ndarray):
    """The offline weight path: (trits int8 [N, K], scales fp16 bits [N, K/128]).

    Rows of W are rotated block-wise by R = (1/32) H_1024 S, then every
    128-group takes the threshold (of 40 candidates, (j/20) mean|v|) and
    least-squares FP16 scale with the smallest reconstruction error."""
    w = np.ascontiguousarray(W, dtype=np.float64)
    s = np.ascontiguousarray(sign, dtype=np.int8)
    N, K = w.shape
    t = np.zeros((N, K), dtype=np.int8)
    sc = np.zeros((N, K // GROUP), dtype=np.uint16)
    _check(_load().oracle_ternarize(_ptr(w), _ptr(s), N, K, _ptr(t), _ptr(sc)), "ternarize")
    return t, sc
