"""Build libbt.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libbt.so")
SOURCES = ["bt_api.cu", "bt_pack.cu", "bt_fwht.cu", "bt_gemv.cu", "bt_gemv_lut.cu", "bt_gemm.cu", "bt_ternarize.cu"]
HEADERS = ["bt_internal.cuh", "bt_slots.cuh", os.path.join("..", "..", "include", "bt.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr", "-Xptxas", "-v", "-Xlinker", "--no-undefined",
]


# Test-only twin of the library: the table-lookup GEMV leaves out one TMA copy
# and every barrier wait gives up after 4096 tries, so a test can watch the
# bounded wait run out (BT_DEVERR_TIMEOUT) without faulting or hanging the GPU.
# Nothing but that test loads it.
WAITTEST_LIB = os.path.join(HERE, "libbt_waittest.so")
WAITTEST_FLAGS = ["-DBT_TEST_WITHHOLD_COPY", "-DBT_SPIN_LIMIT=4096u", "-DBT_WAIT_NS=20000000ull"]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _nvcc(lib: str, extra: list, log_name: str, verbose: bool) -> str:
    cmd = [NVCC, *FLAGS, *extra, *[os.path.join(CSRC, s) for s in SOURCES], "-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    with open(os.path.join(HERE, log_name), "w") as f:
        f.write(" ".join(cmd) + "\n" + log)
    if res.returncode != 0:
        sys.stderr.write(log)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(log)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale(LIB):
        _nvcc(LIB, [], "build.log", verbose)
    return LIB


def build_waittest(force: bool = False) -> str:
    if force or _stale(WAITTEST_LIB):
        _nvcc(WAITTEST_LIB, WAITTEST_FLAGS, "build_waittest.log", False)
    return WAITTEST_LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    build_waittest(force="--force" in sys.argv)
