"""The allocation-free GEMM entry point, w4a16_gemm_noalloc.

Some callers cannot allocate device memory where they run the GEMM (plug-ins of
inference runtimes that forbid allocation after set-up, C callers without a caching
allocator); this entry point uses the library's fixed per-device scratch instead of a
caller workspace.  Here it is called through the C ABI, twice in a row (every call reuses
the same scratch), and each result is compared element by element with the CPU oracle's
fp32 product and with the workspace entry point's output.  This file is collected last so
a failure here cannot hide the other tests.
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


def _layer(M, N, K, g=128):
    import torch
    rng = np.random.default_rng(M * 101 + N + K)
    X, W, s, s_inv = random_layer(rng, M, N, K)
    q, scales, zeros = oracle.quantize_weights(W, s, g)
    d = {"Xd": dev_bits(X, torch.float16), "qw": dev(oracle.pack_device(q).view(np.int32)),
         "sc": dev_bits(scales, torch.float16), "zr": dev_bits(zeros, torch.float16),
         "si": dev(s_inv)}
    Y_ref = oracle.reference_y(X, s_inv, q, scales, zeros, g)
    return d, Y_ref


def _run_noalloc(d, M, N, g=128):
    import torch
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    assert _noalloc_c(d["Xd"], d["qw"], d["sc"], d["zr"], g, d["si"], Y) == w4.W4_OK
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    return to_f64(Y)


# M = 17..32 (four token tiles) is the largest case the 8 MiB scratch holds on 148 SMs.
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (7, 1536, 2048), (16, 12288, 4096),
                                   (17, 4096, 4096), (32, 11008, 4096)])
def test_noalloc_matches_oracle_twice(M, N, K):
    skip_without_gpu()
    g = 128
    d, Y_ref = _layer(M, N, K, g)
    Y_ws = to_f64(w4.w4a16_gemm(d["Xd"], d["qw"], d["sc"], d["zr"], g, s_inv=d["si"]))
    for _ in range(2):
        Y = _run_noalloc(d, M, N, g)
        check_y(Y, Y_ref, "fp16")          # parity with the oracle
        check_y(Y, Y_ws, "fp16")           # and with the workspace entry point


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """M = 33 needs eight token tiles of split-K slots (about 9.7 MB on 148 SMs), more
    than the fixed scratch holds, so the scratch refuses it (the workspace entry point,
    whose decode kernel goes to M = 64, runs it)."""
    skip_without_gpu()
    import torch
    K, N, g = 1024, 256, 128
    M = 33
    X = torch.zeros(M, K, dtype=torch.float16, device="cuda")
    qw = torch.zeros(N * K // 8, dtype=torch.int32, device="cuda")
    sc = torch.ones(K // g, N, dtype=torch.float16, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    s_inv = torch.ones(K, dtype=torch.float32, device="cuda")
    assert _noalloc_c(X, qw, sc, sc, g, s_inv, Y) == w4.W4_ERR_UNSUPPORTED
    # the same sizes through the workspace entry point are fine
    w4.w4a16_gemm(X, qw, sc, sc, g, s_inv=s_inv, Y=Y)
    torch.cuda.synchronize()
    w4.w4_check_device_error()


def _scratch(plant):
    n = ctypes.c_uint64(0)
    assert w4.lib().w4_selftest_noalloc_scratch(int(plant), ctypes.byref(n)) == w4.W4_OK
    return n.value


def test_noalloc_recovers_after_a_timed_out_call():
    """A kernel that gives up a bounded wait can leave flagged split-K partials in the
    shared scratch, which a later call could add into Y.  The test plants such stale words
    (a test aid writes them; nothing faults), lets a bounded wait expire (the watchdog's
    self-test kernel), and checks that w4_check_device_error reports the timeout and
    leaves no nonzero word in the scratch, and that the next two calls match the oracle."""
    skip_without_gpu()
    M, N, K, g = 1, 4096, 4096, 128
    d, Y_ref = _layer(M, N, K, g)
    _run_noalloc(d, M, N, g)                       # scratch set up, device clean
    assert _scratch(plant=False) == 0              # every call leaves it zeroed
    planted = _scratch(plant=True)
    assert planted > 0 and _scratch(plant=False) == planted
    w4.w4_set_wait_limit_ns(2_000_000)
    try:
        w4.w4_selftest_expired_wait()
        with pytest.raises(w4.W4Error) as e:
            w4.w4_check_device_error()
        assert e.value.status == w4.W4_ERR_TIMEOUT
    finally:
        w4.w4_set_wait_limit_ns(2_000_000_000)
    assert _scratch(plant=False) == 0
    for _ in range(2):
        check_y(_run_noalloc(d, M, N, g), Y_ref, "fp16")
