"""Helpers shared by the GPU parity tests (marshalling only)."""
import numpy as np
import torch

import synthetic as S


def dev16(bits: np.ndarray) -> torch.Tensor:
    """uint16 BF16 bit patterns -> CUDA bf16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def host16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy().view(np.uint8)


def section_view(blob, name, dtype):
    return host8(blob.section(name)).view(dtype)


# GEMM tolerance.  The stated bound is a maximum relative error of 2e-3
# against the fp32-accumulated reference over BF16 operands.  It applies
# element-wise to float32 outputs, with a floor of 1e-2 * rms(R) so that
# outputs near zero are judged against the matrix's scale; the floor grows in
# proportion to K / 4096 beyond K = 4096, because the rounding left in an
# output that cancels to near zero is that of its long fp32 reduction (the
# tensor cores do not round every addition to nearest, so it can grow with
# the number of terms, not with their square root).  A BF16 output
# additionally carries its own rounding, up to 2^-8 relative (half an ulp of
# an 8-bit significand).
REL = 2e-3


def gemm_floor(R: np.ndarray, K: int) -> float:
    if not R.size:
        return 0.0
    return 1e-2 * float(np.sqrt(np.mean(R * R))) * max(1.0, K / 4096.0)


def check_gemm(Y: np.ndarray, R: np.ndarray, bf16_out: bool, K: int = 4096):
    R = np.asarray(R, np.float64)
    Y = np.asarray(Y, np.float64)
    floor = gemm_floor(R, K)
    tol = REL * np.maximum(np.abs(R), floor)
    if bf16_out:
        tol = tol + 2.0 ** -8 * np.abs(R)
    err = np.abs(Y - R)
    bad = err > tol
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outside tolerance; worst "
                           f"{float((err / np.maximum(tol, 1e-30)).max()):.3g}x")
    rel = float((err / np.maximum(np.abs(R), floor)).max()) if R.size else 0.0
    return rel


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return S.bits_to_float(bits)


def oracle_gemm(X: np.ndarray, W: np.ndarray, acc: str = "f32") -> np.ndarray:
    """The oracle's R = X . W^T over column blocks of R, one thread per block
    (the oracle's loops release the interpreter lock), so that full-size
    references finish in seconds.  Every element is still the oracle's own
    ascending-k sum."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    X = np.ascontiguousarray(X, np.uint16)
    W = np.ascontiguousarray(W, np.uint16)
    M, N = X.shape[0], W.shape[0]
    R = np.empty((M, N), np.float64)
    nt = max(1, os.cpu_count() or 1)
    step = max(1, -(-N // (4 * nt)))
    bounds = [(n0, min(N, n0 + step)) for n0 in range(0, N, step)]

    def work(b):
        R[:, b[0]:b[1]] = O.gemm(X, W[b[0]:b[1]], acc)

    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(work, bounds))
    return R


def check_swiglu(H: np.ndarray, G: np.ndarray, U: np.ndarray, bf16_out: bool):
    """H = silu(G) * U against the oracle's fp32-accumulated products G, U.
    Each product is allowed the GEMM tolerance (REL with the 1e-2 rms floor);
    that tolerance is carried through h = silu(g) u to first order
    (|silu'(g)| |u| dg + |silu(g)| du, plus the dg du term), and a BF16 output
    adds its rounding (2^-8 relative).  A 1e-5 relative term covers the fp32
    evaluation of the exponential on the device."""
    from oracle import oracle as O
    G = np.asarray(G, np.float64)
    U = np.asarray(U, np.float64)
    H = np.asarray(H, np.float64)
    ref = O.swiglu(G, U)
    fg = 1e-2 * np.sqrt(np.mean(G * G)) if G.size else 0.0
    fu = 1e-2 * np.sqrt(np.mean(U * U)) if U.size else 0.0
    dg = REL * np.maximum(np.abs(G), fg)
    du = REL * np.maximum(np.abs(U), fu)
    sig = 1.0 / (1.0 + np.exp(-np.clip(G, -700, 700)))
    silu = G * sig
    dsilu = sig * (1.0 + G * (1.0 - sig))
    tol = np.abs(dsilu) * np.abs(U) * dg + np.abs(silu) * du + 1.1 * dg * du + 1e-5 * np.abs(ref)
    if bf16_out:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(H - ref)
    bad = err > tol
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outside tolerance; worst "
                           f"{float((err / np.maximum(tol, 1e-30)).max()):.3g}x")
