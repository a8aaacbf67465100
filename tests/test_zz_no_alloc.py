"""The allocation-free GEMM entry point, w4a16_gemm_noalloc.

Some callers cannot allocate device memory where they run the GEMM (plug-ins of
inference runtimes that forbid allocation after set-up, C callers without a caching
allocator); this entry point uses the library's fixed per-device scratch instead of a
caller workspace.  Here it is called through the C ABI and its output is compared with
the workspace entry point's, twice in a row, since every call reuses the same scratch.
This file is collected last so a failure here cannot hide the other tests.
"""
import ctypes

import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from tests.gpu_util import check_y, dev, dev_bits, random_layer, skip_without_gpu, to_f64

pytestmark = pytest.mark.gpu


def _noalloc_c(X, qw, sc, zr, g, s_inv, Y):
    import torch
    L = w4.lib()
    return L.w4a16_gemm_noalloc(
        ctypes.c_void_p(X.data_ptr()), w4.W4_F16, X.shape[0], Y.shape[1], X.shape[1],
        ctypes.c_void_p(qw.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
        ctypes.c_void_p(zr.data_ptr()), None, g, ctypes.c_void_p(s_inv.data_ptr()),
        ctypes.c_void_p(Y.data_ptr()), w4.W4_F16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (7, 1536, 2048), (16, 12288, 4096)])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K):
    skip_without_gpu()
    import torch
    g = 128
    rng = np.random.default_rng(M * 101 + N + K)
    X, W, s, s_inv = random_layer(rng, M, N, K)
    q, scales, zeros = oracle.quantize_weights(W, s, g)
    Xd = dev_bits(X, torch.float16)
    qw = dev(oracle.pack_device(q).view(np.int32))
    sc = dev_bits(scales, torch.float16)
    zr = dev_bits(zeros, torch.float16)
    si = dev(s_inv)
    Y_ws = to_f64(w4.w4a16_gemm(Xd, qw, sc, zr, g, s_inv=si))
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc_c(Xd, qw, sc, zr, g, si, Y) == w4.W4_OK
        torch.cuda.synchronize()
        w4.w4_check_device_error()
        check_y(to_f64(Y), Y_ws, "fp16")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    skip_without_gpu()
    import torch
    K, N, g = 1024, 256, 128
    X = torch.zeros(65, K, dtype=torch.float16, device="cuda")
    qw = torch.zeros(N * K // 8, dtype=torch.int32, device="cuda")
    sc = torch.ones(K // g, N, dtype=torch.float16, device="cuda")
    Y = torch.empty(65, N, dtype=torch.float16, device="cuda")
    s_inv = torch.ones(K, dtype=torch.float32, device="cuda")
    assert _noalloc_c(X, qw, sc, sc, g, s_inv, Y) == w4.W4_ERR_UNSUPPORTED
