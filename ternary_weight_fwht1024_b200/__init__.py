"""Python binding of libbt.so (ternary-weight FWHT-1024 GEMV / GEMM for B200).

Argument marshalling only: every step of the path runs in the CUDA kernels of
libbt.so, called through its C ABI (include/bt.h) with raw device pointers
and the current torch CUDA stream. PyTorch provides device memory and
streams. There is no fallback: if libbt.so is missing or no CUDA device is
present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbt.so")

LAYOUT_B3 = 0
LAYOUT_2BIT = 1
LAYOUT_B3C = 2   # continuous base-3 (no per-group byte padding); bt_pack/unpack and single-row products
F32 = 0
BF16 = 1

DEVERR_INVALID_TRIT = 0x1
DEVERR_INVALID_CODE = 0x2
DEVERR_INVALID_PAD = 0x4
DEVERR_TIMEOUT = 0x8

# Exported entry points, as declared in include/bt.h.
SYMBOLS = (
    "bt_status_string", "bt_version", "bt_codes_row_bytes", "bt_pack", "bt_unpack",
    "bt_fwht1024", "bt_gemv_workspace_bytes", "bt_gemv", "bt_gemv_batched_workspace_bytes", "bt_gemv_batched",
    "bt_gemv_noalloc", "bt_gemm_workspace_bytes", "bt_gemm", "bt_ternarize_workspace_bytes", "bt_ternarize",
)


class GemvProblem(ctypes.Structure):
    """bt_gemv_problem (include/bt.h)."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("x_dtype", ctypes.c_int32), ("x_from", ctypes.c_int32), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64)]

_lock = threading.Lock()
_lib = None
_workspaces: dict = {}


class BtError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libbt.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"libbt.so not built ({LIB_PATH}); run __graft_entry__.build()")
            lib = ctypes.CDLL(LIB_PATH)
            P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
            lib.bt_status_string.argtypes = [I]
            lib.bt_status_string.restype = ctypes.c_char_p
            lib.bt_version.restype = I
            lib.bt_codes_row_bytes.argtypes = [I, I64]
            lib.bt_codes_row_bytes.restype = I64
            lib.bt_pack.argtypes = [I, P, I64, I64, P, P, P]
            lib.bt_unpack.argtypes = [I, P, I64, I64, P, P, P]
            lib.bt_fwht1024.argtypes = [P, P, I64, I64, I, P, P]
            lib.bt_gemv_workspace_bytes.argtypes = [I, I64, I64, I64]
            lib.bt_gemv_workspace_bytes.restype = SZ
            lib.bt_gemv.argtypes = [I, P, P, P, I, P, I64, I64, I64, I, P, P, SZ, P, P]
            lib.bt_gemv_noalloc.argtypes = [I, P, P, P, I, P, I64, I64, I64, I, P, P, P]
            PP = ctypes.POINTER(GemvProblem)
            lib.bt_gemv_batched_workspace_bytes.argtypes = [I, PP, I]
            lib.bt_gemv_batched_workspace_bytes.restype = SZ
            lib.bt_gemv_batched.argtypes = [I, PP, I, P, I, P, SZ, P, P]
            lib.bt_gemm_workspace_bytes.argtypes = [I, I64, I64, I64]
            lib.bt_gemm_workspace_bytes.restype = SZ
            lib.bt_gemm.argtypes = [I, P, P, P, I, P, I64, I64, I64, P, P, SZ, P, P]
            lib.bt_ternarize_workspace_bytes.argtypes = [I64, I64]
            lib.bt_ternarize_workspace_bytes.restype = SZ
            lib.bt_ternarize.argtypes = [P, P, I64, I64, P, P, P, SZ, P]
            for name in ("bt_pack", "bt_unpack", "bt_fwht1024", "bt_gemv", "bt_gemv_batched", "bt_gemv_noalloc",
                         "bt_gemm", "bt_ternarize"):
                getattr(lib, name).restype = I
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().bt_status_string(status).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise BtError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("libbt takes CUDA tensors only")


def codes_row_bytes(layout: int, K: int) -> int:
    return int(load().bt_codes_row_bytes(layout, K))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A cached uint8 workspace of at least nbytes on `device`, one per stream
    (scratch: the library expects no particular contents)."""
    key = (torch.device(device), torch.cuda.current_stream(device).cuda_stream)
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    return buf


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A workspace of its own."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def pack(trits: torch.Tensor, layout: int = LAYOUT_B3, dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """int8 [N, K] trits -> uint8 [N, row bytes] codes."""
    _require_cuda(trits, dev_err)
    t = trits.contiguous()
    N, K = t.shape
    codes = torch.empty((N, max(codes_row_bytes(layout, K), 0) if K else 0), dtype=torch.uint8, device=t.device)
    _check("bt_pack", load().bt_pack(layout, _ptr(t), N, K, _ptr(codes), _ptr(dev_err), _stream(t.device)))
    return codes


def unpack(codes: torch.Tensor, K: int, layout: int = LAYOUT_B3,
           dev_err: torch.Tensor | None = None) -> torch.Tensor:
    _require_cuda(codes, dev_err)
    c = codes.contiguous()
    N = c.shape[0]
    trits = torch.empty((N, K), dtype=torch.int8, device=c.device)
    _check("bt_unpack", load().bt_unpack(layout, _ptr(c), N, K, _ptr(trits), _ptr(dev_err), _stream(c.device)))
    return trits


def fwht1024(x: torch.Tensor, sign: torch.Tensor, out_dtype: int = F32,
             out: torch.Tensor | None = None) -> torch.Tensor:
    """x' = (1/32) H_1024 (S . x) per 1024-block; x bf16 [M, K]."""
    _require_cuda(x, sign, out)
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    xc = x.contiguous()
    M, K = xc.shape
    if out is None:
        out = torch.empty((M, K), dtype=torch.float32 if out_dtype == F32 else torch.bfloat16, device=x.device)
    elif out.dtype != (torch.float32 if out_dtype == F32 else torch.bfloat16) or tuple(out.shape) != (M, K) \
            or not out.is_contiguous():
        raise ValueError("out must be a contiguous [M, K] tensor of the output dtype")
    _check("bt_fwht1024", load().bt_fwht1024(_ptr(xc), _ptr(sign), M, K, out_dtype, _ptr(out), _stream(x.device)))
    return out


def _x_dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return BF16
    if x.dtype == torch.float32:
        return F32
    raise TypeError("x must be bfloat16 or float32")


def gemv_workspace_bytes(layout: int, M: int, N: int, K: int) -> int:
    return int(load().bt_gemv_workspace_bytes(layout, M, N, K))


def gemv(codes: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, sign: torch.Tensor | None, N: int,
         layout: int = LAYOUT_B3, y_dtype: int = F32, out: torch.Tensor | None = None,
         ws: torch.Tensor | None = None, dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """y [M, N] = x' W^T for 1 <= M <= 16; x' = R x when `sign` is given."""
    _require_cuda(codes, scales, x, sign, out, ws, dev_err)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if y_dtype == F32 else torch.bfloat16, device=x.device)
    need = gemv_workspace_bytes(layout, M, N, K)
    if ws is None:
        ws = workspace(need, x.device)
    _check("bt_gemv", load().bt_gemv(layout, _ptr(codes), _ptr(scales), _ptr(x), _x_dtype(x), _ptr(sign),
                                      M, N, K, y_dtype, _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_err),
                                      _stream(x.device)))
    return out


def _problem_array(problems):
    arr = (GemvProblem * len(problems))()
    for i, p in enumerate(problems):
        x = p.get("x")
        x_from = int(p.get("x_from", -1))
        arr[i].codes = p["codes"].data_ptr() if "codes" in p else None  # sizes alone suffice for the workspace query
        arr[i].scales = p["scales"].data_ptr() if "scales" in p else None
        arr[i].x = x.data_ptr() if (x is not None and x_from < 0) else None
        arr[i].x_dtype = _x_dtype(x) if (x is not None and x_from < 0) else BF16
        arr[i].x_from = x_from
        arr[i].y = p["y"].data_ptr() if "y" in p else None
        arr[i].N = int(p["N"])
        arr[i].K = int(p["K"])
    return arr


def gemv_batched_workspace_bytes(layout: int, problems) -> int:
    arr = _problem_array(problems)
    return int(load().bt_gemv_batched_workspace_bytes(layout, arr, len(problems)))


def gemv_batched(problems, sign: torch.Tensor | None, layout: int = LAYOUT_B3, y_dtype: int = F32,
                 ws: torch.Tensor | None = None, dev_err: torch.Tensor | None = None):
    """y_p = W_p (R x_p) for a list of single-row problems: one persistent
    kernel per group of up to 12 matrices (a matrix reading an output of the
    current group starts the next group), then the reductions that write y.

    Each problem is a dict with codes, scales, y ([1, N] of y_dtype), N, K and
    either x ([1, K] bf16, or f32 when sign is None) or x_from (the index of an
    earlier problem whose y is this x). Returns the list of y tensors."""
    if not problems:
        return []
    dev = problems[0]["y"].device
    for p in problems:
        _require_cuda(p["codes"], p["scales"], p.get("x"), p["y"])
    _require_cuda(sign, ws, dev_err)
    arr = _problem_array(problems)
    need = int(load().bt_gemv_batched_workspace_bytes(layout, arr, len(problems)))
    if ws is None:
        ws = workspace(need, dev)
    _check("bt_gemv_batched", load().bt_gemv_batched(layout, arr, len(problems), _ptr(sign), y_dtype, _ptr(ws),
                                                      ws.numel(), _ptr(dev_err), _stream(dev)))
    return [p["y"] for p in problems]


def gemv_noalloc(codes: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, sign: torch.Tensor | None, N: int,
                 layout: int = LAYOUT_B3, y_dtype: int = F32, out: torch.Tensor | None = None,
                 dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """bt_gemv without a caller-provided workspace (scratch lives in libbt.so).

    For callers that cannot allocate device memory at call time. Calls share
    one 8 MiB scratch array per GPU: calls that may overlap on the GPU race.
    `out` may be passed to avoid allocating the result here as well.
    """
    _require_cuda(codes, scales, x, sign, out, dev_err)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if y_dtype == F32 else torch.bfloat16, device=x.device)
    _check("bt_gemv_noalloc", load().bt_gemv_noalloc(layout, _ptr(codes), _ptr(scales), _ptr(x), _x_dtype(x),
                                                      _ptr(sign), M, N, K, y_dtype, _ptr(out), _ptr(dev_err),
                                                      _stream(x.device)))
    return out


def gemm_workspace_bytes(layout: int, M: int, N: int, K: int) -> int:
    return int(load().bt_gemm_workspace_bytes(layout, M, N, K))


def gemm(codes: torch.Tensor, scales: torch.Tensor, x: torch.Tensor, sign: torch.Tensor | None, N: int,
         layout: int = LAYOUT_B3, out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
         dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """Y bf16 [M, N] = X' W^T on the tcgen05 tensor cores; M, N multiples of 128."""
    _require_cuda(codes, scales, x, sign, out, ws, dev_err)
    M, K = x.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = gemm_workspace_bytes(layout, M, N, K)
    if ws is None:
        ws = workspace(need, x.device)
    _check("bt_gemm", load().bt_gemm(layout, _ptr(codes), _ptr(scales), _ptr(x), _x_dtype(x), _ptr(sign),
                                      M, N, K, _ptr(out), _ptr(ws), ws.numel(), _ptr(dev_err),
                                      _stream(x.device)))
    return out


def ternarize(W: torch.Tensor, sign: torch.Tensor, ws: torch.Tensor | None = None):
    """Offline weight path: float W [N, K] -> (trits int8 [N, K], scales fp16 bits [N, K/128]).

    Rows of W are rotated block-wise by R = (1/32) H_1024 S, then every group
    of 128 takes the threshold and FP16 scale with the smallest reconstruction
    error; pack the trits with pack() and multiply with gemv()/gemm() as usual."""
    _require_cuda(W, sign, ws)
    if W.dtype != torch.float32:
        raise TypeError("W must be float32")
    Wc = W.contiguous()
    N, K = Wc.shape
    trits = torch.empty((N, K), dtype=torch.int8, device=W.device)
    scales = torch.empty((N, K // 128), dtype=torch.int16, device=W.device)
    need = int(load().bt_ternarize_workspace_bytes(N, K))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    _check("bt_ternarize", load().bt_ternarize(_ptr(Wc), _ptr(sign), N, K, _ptr(trits), _ptr(scales), _ptr(ws),
                                                ws.numel(), _stream(W.device)))
    return trits, scales
