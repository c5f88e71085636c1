"""The allocation-free direct-palette GEMM (uw_gemm_direct_palette_noalloc).

It serves callers that cannot allocate device memory when they call the
GEMM -- engines that reserve all memory up front, code that must not risk the
device synchronisation an allocation can cause, plugins that do not own the
allocator.  Its scratch is a fixed array inside the library.  This file is
collected last on purpose; it must pass alone in a fresh process and after
the other tests.  Each case calls the entry point twice in a row through the
C ABI, since the fixed scratch keeps the previous call's contents.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_gemm_bf16_b200 as uw
import synthetic as S
from tests.gpu_util import check_gemm, dev16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blob_and_w():
    W = S.weight_with_verbatim_rows(1000, 1024, seed=41, frac_groups=0.01)
    return uw.uw_compress(dev16(W)), W


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("out_f32", [True, False])
def test_noalloc_matches_workspace_gemm(blob_and_w, M, out_f32):
    blob, W = blob_and_w
    X = dev16(S.activations(M, W.shape[1], seed=500 + M))
    ref = uw.uw_gemm(X, blob, "direct_palette", out_f32=True).double().cpu().numpy()
    L = uw.lib()
    for _ in range(2):
        Y = torch.full((M, blob.N), float("nan"), dtype=torch.float32 if out_f32 else torch.bfloat16,
                       device="cuda")
        st = L.uw_gemm_direct_palette_noalloc(ctypes.c_void_p(X.data_ptr()), M, blob.handle,
                                              ctypes.c_void_p(Y.data_ptr()), 1 if out_f32 else 0,
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, uw.status_str(st)
        torch.cuda.synchronize()
        check_gemm(Y.double().cpu().numpy(), ref, bf16_out=not out_f32)
    assert uw.uw_last_device_status() == 0


def test_noalloc_rejects_batches_beyond_its_scratch(blob_and_w):
    blob, W = blob_and_w
    M = 256
    X = dev16(S.activations(M, W.shape[1], seed=7))
    Y = torch.empty(M, blob.N, dtype=torch.bfloat16, device="cuda")
    st = uw.lib().uw_gemm_direct_palette_noalloc(ctypes.c_void_p(X.data_ptr()), M, blob.handle,
                                                 ctypes.c_void_p(Y.data_ptr()), 0,
                                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 5   # UW_ERR_WORKSPACE, nothing launched
