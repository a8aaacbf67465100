"""Bounded waits: a kernel waiting on a barrier that nothing completes gives up after the
configured limit and reports it through the device error word, leaving the context usable.
No GPU fault, trap or hang is involved."""
import pytest

import bit_weight_only_w4_b200 as w4
from tests.gpu_util import skip_without_gpu

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    skip_without_gpu()
    import torch
    w4.w4_check_device_error()                    # start clean
    w4.w4_set_wait_limit_ns(2_000_000)            # 2 ms
    try:
        w4.w4_selftest_expired_wait()
        with pytest.raises(w4.W4Error) as e:
            w4.w4_check_device_error()
        assert e.value.status == w4.W4_ERR_TIMEOUT
        w4.w4_check_device_error()                # the word was cleared
    finally:
        w4.w4_set_wait_limit_ns(2_000_000_000)
    x = torch.ones(4, device="cuda")              # context still works
    assert float(x.sum()) == 4.0


def test_out_of_range_gidx_is_reported():
    skip_without_gpu()
    import torch
    N, K, g = 16, 64, 32
    W = torch.randn(N, K, dtype=torch.float16, device="cuda") * 0.02
    g_idx = torch.zeros(K, dtype=torch.int32, device="cuda")
    g_idx[5] = 7                                  # only groups 0 and 1 exist
    w4.w4_quantize_pack(W, None, g, True, g_idx)
    with pytest.raises(w4.W4Error) as e:
        w4.w4_check_device_error()
    assert e.value.status == w4.W4_ERR_DEVICE_ARG
