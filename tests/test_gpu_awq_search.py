"""GPU parity of w4_awq_search against the oracle's search: the same chosen candidate (or
two candidates whose losses agree within the tolerance), every loss within 1e-3 relative
(the products differ only in fp32 summation order), and the chosen s equal to the oracle's
up to the last fp32 bits of exp; the decode and the prefill GEMM paths, fp16 and bf16
calibration rows."""
import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from tests.gpu_util import dev_bits, skip_without_gpu

pytestmark = pytest.mark.gpu


def layer(rng, M, N, K, act="fp16"):
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, size=max(1, K // 100), replace=False)] *= 20
    W = (rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)).astype(np.float16)
    X = x.astype(np.float16).view(np.uint16) if act == "fp16" else oracle.f32_to_bf16(x)
    return X, W.view(np.uint16)


def run(X, W, g, sym, n_grid, act="fp16"):
    import torch
    tdt = torch.float16 if act == "fp16" else torch.bfloat16
    best, a, losses, s = w4.w4_awq_search(dev_bits(W, torch.float16), dev_bits(X, tdt), g, sym, n_grid)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    assert a == best / n_grid
    return best, losses, s.cpu().numpy()


@pytest.mark.parametrize("M,N,K,g,sym,n_grid,act", [
    (32, 256, 512, 128, False, 8, "fp16"),     # decode GEMM path
    (100, 256, 512, 64, True, 6, "fp16"),      # prefill GEMM path
    (16, 128, 256, 32, False, 5, "bf16"),      # bf16 calibration rows
])
def test_search_matches_oracle(M, N, K, g, sym, n_grid, act):
    skip_without_gpu()
    rng = np.random.default_rng(M + N + K + g)
    X, W = layer(rng, M, N, K, act)
    best, losses, s = run(X, W, g, sym, n_grid, act)
    o_best, o_losses, o_s = oracle.awq_search(W, X, g, sym, n_grid, x_is_bf16=(act == "bf16"))
    rel = np.abs(losses - o_losses) / o_losses
    assert rel.max() <= 1e-3, (losses, o_losses)
    if best != o_best:
        assert abs(o_losses[best] - o_losses[o_best]) <= 1e-3 * o_losses[o_best]
    else:
        assert np.allclose(s, o_s, rtol=1e-6, atol=0)
    assert best > 0                              # salient channels: AWQ beats plain RTN


def test_search_equal_magnitudes_gives_unit_scales():
    skip_without_gpu()
    rng = np.random.default_rng(9)
    M, N, K, g = 8, 128, 256, 64
    X = (rng.choice([-1.0, 1.0], size=(M, K)) * 0.5).astype(np.float16).view(np.uint16)
    _, W = layer(rng, M, N, K)
    best, losses, s = run(X, W, g, False, 4)
    assert best == 0
    assert np.all(s == np.float32(1))
    assert np.all(losses == losses[0])


def test_gemm_after_search_is_unaffected():
    """The search uses a workspace of its own: a decode GEMM through the binding's cached
    workspace right after it still matches the oracle."""
    skip_without_gpu()
    import torch
    from tests.gpu_util import check_y, dev, to_f64
    rng = np.random.default_rng(21)
    X, W = layer(rng, 16, 256, 512)
    run(X, W, 128, False, 3)
    q, sc, zr = oracle.quantize_weights(W, None, 128, False)
    Xd = dev_bits(X[:3], torch.float16)
    Y = w4.w4a16_gemm(Xd, dev(oracle.pack_device(q).view(np.int32)), dev_bits(sc, torch.float16),
                      dev_bits(zr, torch.float16), 128)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    check_y(to_f64(Y), oracle.reference_y(X[:3], None, q, sc, zr, 128), "fp16")
