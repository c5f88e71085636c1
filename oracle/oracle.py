"""CPU oracle for the Unweight-style BF16 weight format -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product library never calls it, and
it never calls the product library: it is a plain statement of what the GPU
path must compute, written from the web page "Cloudflare推出Unweight無損壓縮系統，
將LLM模型大小壓縮15-22%" (easyvibecoding.app), §BF16權重壓縮原理, §四種執行管道 and
§重建矩陣乘法核心運作.

The arithmetic lives in ``uw_oracle.c`` (plain loops, one function per step);
this file only marshals numpy arrays into those functions, in the order of the
method:

  split -> histogram -> palette -> verbatim groups -> symbols -> index plane
  -> verbatim store -> frequencies -> code lengths -> canonical codes
  -> encode (stream + chunk offsets)

and back (decode -> exponents -> BF16), plus the reference product
R = X . W^T accumulated in float64 (or float32 in ascending k), and the
SwiGLU that joins the gate and up products, H = silu(G) * U.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "uw_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GROUP = 64
PALETTE = 16
SEG = 256
CHUNK_SEGS = 16
LMAX = 12


def build(force: bool = False) -> str:
    """Compile uw_oracle.c with gcc (plain -O2, no vectorisation flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L = _lib
        L.or_split.argtypes = [P, I64, P, P]
        L.or_merge.argtypes = [P, P, I64, P]
        L.or_histogram.argtypes = [P, I64, P]
        L.or_palette.argtypes = [P, P, P]
        L.or_verbatim.argtypes = [P, P, I64, I64, P]
        L.or_verbatim.restype = I64
        L.or_symbols.argtypes = [P, P, P, I64, I64, P]
        L.or_index_plane.argtypes = [P, I64, P]
        L.or_verbatim_store.argtypes = [P, P, I64, I64, P, P, P, P]
        L.or_frequencies.argtypes = [P, I64, P]
        L.or_code_lengths.argtypes = [P, ctypes.c_int, P]
        L.or_code_lengths.restype = ctypes.c_int
        L.or_canonical_codes.argtypes = [P, P]
        L.or_stream_bits.argtypes = [P, I64, P]
        L.or_stream_bits.restype = ctypes.c_uint64
        L.or_encode.argtypes = [P, I64, P, P, P, I64, P, P]
        L.or_decode_symbols.argtypes = [P, I64, P, ctypes.c_uint64, I64, P]
        L.or_decode_symbols.restype = ctypes.c_uint64
        L.or_exponents_from_symbols.argtypes = [P, I64, P, P, P, P, P]
        L.or_gemm.argtypes = [P, P, I64, I64, I64, ctypes.c_int, P]
        L.or_gemm_one.argtypes = [P, P, I64, I64, I64, ctypes.c_int]
        L.or_gemm_one.restype = ctypes.c_double
        L.or_swiglu.argtypes = [P, P, I64, P]
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Individual steps (thin wrappers; each names the step of uw_oracle.c).
# --------------------------------------------------------------------------
def split(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    e = np.empty(w.size, np.uint8)
    sm = np.empty(w.size, np.uint8)
    lib().or_split(_p(w), w.size, _p(e), _p(sm))
    return e, sm


def merge(e: np.ndarray, sm: np.ndarray) -> np.ndarray:
    e = np.ascontiguousarray(e, np.uint8).reshape(-1)
    sm = np.ascontiguousarray(sm, np.uint8).reshape(-1)
    w = np.empty(e.size, np.uint16)
    lib().or_merge(_p(e), _p(sm), e.size, _p(w))
    return w


def histogram(e: np.ndarray) -> np.ndarray:
    e = np.ascontiguousarray(e, np.uint8).reshape(-1)
    h = np.zeros(256, np.uint64)
    lib().or_histogram(_p(e), e.size, _p(h))
    return h


def palette(hist: np.ndarray):
    hist = np.ascontiguousarray(hist, np.uint64)
    pal = np.zeros(PALETTE, np.uint8)
    inv = np.zeros(256, np.uint8)
    lib().or_palette(_p(hist), _p(pal), _p(inv))
    return pal, inv


def verbatim(e, inv, N, K):
    verb = np.zeros(N * K // GROUP, np.uint8)
    V = lib().or_verbatim(_p(e), _p(inv), N, K, _p(verb))
    return verb, int(V)


def symbols(e, inv, verb, N, K):
    s = np.empty(N * K, np.uint8)
    lib().or_symbols(_p(e), _p(inv), _p(verb), N, K, _p(s))
    return s


def index_plane(s):
    idx = np.empty(s.size // 2, np.uint8)
    lib().or_index_plane(_p(s), s.size, _p(idx))
    return idx


def verbatim_store(verb, e, N, K, V):
    G = N * K // GROUP
    GW = (G + 31) // 32
    NW = 4 * ((N + 127) // 128)
    vbits = np.zeros(GW, np.uint32)
    vpre = np.zeros(GW, np.uint32)
    vexp = np.zeros(V * GROUP, np.uint8)
    vcol = np.zeros((K // GROUP) * NW, np.uint32)
    lib().or_verbatim_store(_p(verb), _p(e), N, K, _p(vbits), _p(vpre), _p(vexp), _p(vcol))
    return vbits, vpre, vexp, vcol


def frequencies(s):
    f = np.zeros(PALETTE, np.uint64)
    lib().or_frequencies(_p(s), s.size, _p(f))
    return f


def code_lengths(freq, lmax: int = LMAX):
    freq = np.ascontiguousarray(freq, np.uint64)
    assert freq.size == PALETTE
    ln = np.zeros(PALETTE, np.uint8)
    rc = lib().or_code_lengths(_p(freq), int(lmax), _p(ln))
    if rc != 0:
        raise ValueError("symbols do not fit the length limit")
    return ln


def canonical_codes(lengths):
    lengths = np.ascontiguousarray(lengths, np.uint8)
    codes = np.zeros(PALETTE, np.uint32)
    lib().or_canonical_codes(_p(lengths), _p(codes))
    return codes


def encode(s, lengths, codes):
    bits = int(lib().or_stream_bits(_p(s), s.size, _p(lengths)))
    nwords = (bits + 31) // 32 + 2
    nseg = (s.size + SEG - 1) // SEG
    nchunk = (nseg + CHUNK_SEGS - 1) // CHUNK_SEGS
    stream = np.zeros(nwords, np.uint32)
    chunk_off = np.zeros(nchunk, np.uint64)
    seg_rel = np.zeros(nseg, np.uint16)
    lib().or_encode(_p(s), s.size, _p(lengths), _p(codes), _p(stream), nwords,
                    _p(chunk_off), _p(seg_rel))
    return stream, chunk_off, seg_rel, bits


def decode_symbols(stream, lengths, start_bit: int, count: int):
    out = np.zeros(count, np.uint8)
    end = lib().or_decode_symbols(_p(stream), stream.size, _p(np.ascontiguousarray(lengths, np.uint8)),
                                  int(start_bit), int(count), _p(out))
    if end == np.iinfo(np.uint64).max:
        raise ValueError("undecodable bit pattern")
    return out, int(end)


# --------------------------------------------------------------------------
# Whole-matrix compress and decodes.
# --------------------------------------------------------------------------
def compress(W: np.ndarray) -> dict:
    """All format sections for a row-major BF16 matrix W[N, K] (uint16 bits)."""
    W = np.ascontiguousarray(W, np.uint16)
    N, K = W.shape
    if N < 1 or K < GROUP or K % GROUP:
        raise ValueError("need N >= 1 and K a positive multiple of 64")
    e, sm = split(W)
    hist = histogram(e)
    pal, inv = palette(hist)
    verb, V = verbatim(e, inv, N, K)
    s = symbols(e, inv, verb, N, K)
    idx = index_plane(s)
    vbits, vpre, vexp, vcol = verbatim_store(verb, e, N, K, V)
    freq = frequencies(s)
    lengths = code_lengths(freq, LMAX)
    codes = canonical_codes(lengths)
    stream, chunk_off, seg_rel, bits = encode(s, lengths, codes)
    return dict(N=N, K=K, G=N * K // GROUP, V=V, hist=hist, palette=pal, inv=inv,
                verb=verb, symbols=s, sm=sm, idx=idx, vbits=vbits, vpre=vpre,
                vexp=vexp, vcol=vcol, freq=freq, code_len=lengths, codes=codes,
                stream=stream, chunk_off=chunk_off, seg_rel=seg_rel, total_bits=bits)


def decode_all_symbols(blob: dict) -> np.ndarray:
    s, _ = decode_symbols(blob["stream"], blob["code_len"], 0, blob["N"] * blob["K"])
    return s


def exponents(blob: dict, s: np.ndarray) -> np.ndarray:
    n = s.size
    out = np.empty(n, np.uint8)
    lib().or_exponents_from_symbols(_p(s), n, _p(blob["palette"]), _p(blob["vbits"]),
                                    _p(blob["vpre"]), _p(blob["vexp"]) if blob["vexp"].size else None,
                                    _p(out))
    return out


def decode_exponent(blob: dict) -> np.ndarray:
    """Exponent-only decode: the exponent byte of every weight."""
    return exponents(blob, decode_all_symbols(blob))


def decode_full(blob: dict) -> np.ndarray:
    """Full decode: the original BF16 bit patterns, shape [N, K]."""
    e = decode_exponent(blob)
    return merge(e, blob["sm"]).reshape(blob["N"], blob["K"])


def transcode(blob: dict) -> np.ndarray:
    """Palette transcode: the 4-bit index plane rebuilt from the stream."""
    return index_plane(decode_all_symbols(blob))


def gemm(X: np.ndarray, W: np.ndarray, acc: str = "f64") -> np.ndarray:
    """R = X . W^T over BF16 bit patterns X[M,K], W[N,K]; float64 result."""
    X = np.ascontiguousarray(X, np.uint16)
    W = np.ascontiguousarray(W, np.uint16)
    M, K = X.shape
    N, K2 = W.shape
    assert K == K2
    R = np.zeros((M, N), np.float64)
    lib().or_gemm(_p(X), _p(W), M, N, K, 1 if acc == "f64" else 0, _p(R))
    return R


def gemm_one(X: np.ndarray, W: np.ndarray, m: int, n: int, acc: str = "f64") -> float:
    X = np.ascontiguousarray(X, np.uint16)
    W = np.ascontiguousarray(W, np.uint16)
    return float(lib().or_gemm_one(_p(X), _p(W), X.shape[1], int(m), int(n), 1 if acc == "f64" else 0))


def swiglu(G: np.ndarray, U: np.ndarray) -> np.ndarray:
    """H = silu(G) * U elementwise (float64), silu(z) = z / (1 + e^-z)."""
    G = np.ascontiguousarray(G, np.float64)
    U = np.ascontiguousarray(U, np.float64)
    assert G.shape == U.shape
    H = np.empty_like(G)
    lib().or_swiglu(_p(G), _p(U), G.size, _p(H))
    return H
