"""The allocation-free direct-palette GEMM (uw_gemm_direct_palette_noalloc).

It serves callers that cannot allocate device memory when they call the
GEMM -- engines that reserve all memory up front, code that must not risk the
device synchronisation an allocation can cause, plugins that do not own the
allocator.  Its scratch is a fixed array inside the library.  This file is
collected last on purpose; it must pass alone in a fresh process and after
the other tests.  Each case calls the entry point twice in a row through the
C ABI, since the fixed scratch keeps the previous call's contents, and
compares every output with the CPU oracle's fp32-accumulated product.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_gemm_bf16_b200 as uw
import synthetic as S
from oracle import oracle as O
from tests.gpu_util import check_gemm, dev16

pytestmark = pytest.mark.gpu

SHAPES = {
    # 8 row tiles: batch 1 runs the CUDA-core GEMV (no scratch), 5 and 16 the
    # tensor cores with stream-K partial sums in the fixed scratch
    "1000x1024": lambda: S.weight_with_verbatim_rows(1000, 1024, seed=41, frac_groups=0.01),
    # 80 row tiles: batch 1 stays on the tensor cores (stream-K, scratch used)
    "10240x512": lambda: S.weight_with_verbatim_rows(10240, 512, seed=42, frac_groups=0.01),
}
_cache = {}


def _case(name):
    if name not in _cache:
        W = SHAPES[name]()
        _cache[name] = (uw.uw_compress(dev16(W)), W)
    return _cache[name]


def _call(X, M, blob, Y, out_f32):
    return uw.lib().uw_gemm_direct_palette_noalloc(ctypes.c_void_p(X.data_ptr()), M, blob.handle,
                                                   ctypes.c_void_p(Y.data_ptr()), 1 if out_f32 else 0,
                                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("shape,M", [("1000x1024", 1), ("1000x1024", 5), ("1000x1024", 16),
                                     ("10240x512", 1), ("10240x512", 16)])
@pytest.mark.parametrize("out_f32", [True, False])
def test_noalloc_matches_oracle(shape, M, out_f32):
    blob, W = _case(shape)
    Xh = S.activations(M, W.shape[1], seed=500 + M)
    X = dev16(Xh)
    R = O.gemm(Xh, W, "f32")
    for _ in range(2):
        Y = torch.full((M, blob.N), float("nan"), dtype=torch.float32 if out_f32 else torch.bfloat16,
                       device="cuda")
        st = _call(X, M, blob, Y, out_f32)
        assert st == 0, uw.status_str(st)
        torch.cuda.synchronize()
        check_gemm(Y.double().cpu().numpy(), R, bf16_out=not out_f32)
    assert uw.uw_last_device_status() == 0


def test_noalloc_rejects_batches_beyond_its_scratch():
    blob, W = _case("1000x1024")
    M = 256
    X = dev16(S.activations(M, W.shape[1], seed=7))
    Y = torch.empty(M, blob.N, dtype=torch.bfloat16, device="cuda")
    assert _call(X, M, blob, Y, False) == 5   # UW_ERR_WORKSPACE, nothing launched
