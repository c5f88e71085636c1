"""Builds libunweight.so (CUDA for sm_100a) in-tree with nvcc."""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libunweight.so")
SOURCES = ["uw_host.cpp", "uw_compress.cu", "uw_decode.cu", "uw_gemm.cu", "uw_gemv.cu"]
HEADERS = ["uw_internal.h", "uw_device.cuh", os.path.join("..", "..", "include", "unweight.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
BUILD_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler",
               "-fvisibility=default", "--expt-relaxed-constexpr"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


STAMP = LIB + ".srchash"


def source_hash() -> str:
    h = hashlib.sha256()
    for f in SOURCES + HEADERS + [os.path.abspath(__file__)]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _strip_comments(text: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed
    (string and character literals kept verbatim)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def code_hash(unit: str | None = None) -> str:
    """Hash of what the compiler sees (sources without comments, plus the
    build flags): measurements keyed to it stay valid across comment edits.
    With `unit` (a source file name), only that translation unit and the
    headers count, so a measurement of its kernels survives changes to the
    other units."""
    h = hashlib.sha256(" ".join(ARCH + BUILD_FLAGS).encode())
    for f in ([unit] if unit else SOURCES) + HEADERS:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(_strip_comments(fh.read()).encode())
    return h.hexdigest()


# translation unit of each measured kernel family
KERNEL_UNITS = {"k_decode": "uw_decode.cu", "k_gemm": "uw_gemm.cu", "k_gemv": "uw_gemv.cu"}


def kernel_code_hash(kernel: str) -> str:
    """code_hash of the unit that defines `kernel` (a profile short name)."""
    for prefix, unit in KERNEL_UNITS.items():
        if kernel.startswith(prefix):
            return code_hash(unit)
    return code_hash()


def stale() -> bool:
    """True when the library is missing or was built from other sources."""
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return True
    with open(STAMP) as fh:
        return fh.read().strip() != source_hash()


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, *BUILD_FLAGS, *extra, *[os.path.join(CSRC, f) for f in SOURCES], "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as fh:
        fh.write(source_hash())
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else ())
    print(LIB)
