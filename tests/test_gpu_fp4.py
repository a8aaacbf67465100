"""GPU parity of the block-scaled FP4 comparator (NVFP4, MXFP4) against the CPU oracle.

Quantisation is integer work and must match bit for bit: the E2M1 codes (read back in
the canonical layout), the block-scale bytes and the NVFP4 tensor scale.  The GEMM is held
to the stated bound (relative L2 1e-3, max-abs 2e-2) against the oracle's fp32 product of
the fp16 activations with the dequantised weights (E2M1 x block scale x tensor scale,
exact in fp64, rounded to fp32).  The GEMM inputs are the oracle's own codes and scales,
so these tests do not depend on the GPU quantiser.
"""
import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from bit_weight_only_w4_b200 import workloads
from tests.gpu_util import check_y, dev, dev_bits, host_u32, skip_without_gpu, to_f64

pytestmark = pytest.mark.gpu

FMTS = ("nvfp4", "mxfp4")


def _weights(rng, N, K, bf16=False):
    W = (rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02))
    return oracle.f32_to_bf16(W) if bf16 else W.astype(np.float16).view(np.uint16)


def _oracle_quant(W_bits, fmt, bf16=False):
    if fmt == "nvfp4":
        codes, bs, gs = oracle.nvfp4_quantize(W_bits, bf16)
        return codes, bs, gs
    codes, es = oracle.mxfp4_quantize(W_bits, bf16)
    return codes, es, None


def _gpu_quant(W_bits, fmt, bf16=False):
    import torch
    Wd = dev_bits(W_bits, torch.bfloat16 if bf16 else torch.float16)
    qw, bs, ts = w4.w4_fp4_quantize_pack(Wd, fmt)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    N, K = W_bits.shape
    canon = w4.w4_unpack_canonical(qw, N, K)
    torch.cuda.synchronize()
    return (host_u32(canon).reshape(N, K // 8), bs.cpu().numpy(),
            None if ts is None else np.float32(ts.cpu().numpy()[0]), qw)


def _check_quant(W_bits, fmt, bf16=False):
    codes, bs, gs = _oracle_quant(W_bits, fmt, bf16)
    canon, gbs, ggs, _ = _gpu_quant(W_bits, fmt, bf16)
    assert np.array_equal(canon, oracle.pack_canonical(codes)), "codes differ"
    assert np.array_equal(gbs, bs.T), "block scales differ"
    if fmt == "nvfp4":
        assert np.float32(ggs).view(np.uint32) == np.float32(gs).view(np.uint32), (ggs, gs)
    else:
        assert ggs is None


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(16, 64), (48, 192), (256, 1024), (1024, 4096)])
@pytest.mark.parametrize("bf16", [False, True])
def test_fp4_quantize_is_bit_exact(fmt, N, K, bf16):
    skip_without_gpu()
    rng = np.random.default_rng(N * 7 + K + bf16)
    _check_quant(_weights(rng, N, K, bf16), fmt, bf16)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp4_quantize_edge_values(fmt):
    """Zero blocks, signed zeros, exact ties of the E2M1 grid, values near the fp16 maximum
    and fp16 subnormals, each in blocks of their own."""
    skip_without_gpu()
    N, K = 32, 256
    rng = np.random.default_rng(3)
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    W[0, :] = 0.0                                  # an all-zero row
    W[1, :32] = -0.0                               # negative zeros
    W[2, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4, np.float32)   # ties x 1
    W[3, :32] = 60000.0 * rng.standard_normal(32).astype(np.float32).clip(-1, 1)
    W[4, :32] = np.float32(2.0 ** -20) * rng.standard_normal(32).astype(np.float32)
    W[5, 32:64] = -W[2, :32]
    _check_quant(W.astype(np.float16).view(np.uint16), fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp4_quantize_all_zero_tensor(fmt):
    skip_without_gpu()
    W = np.zeros((64, 128), np.uint16)
    _check_quant(W, fmt)


def _gemm_case(M, N, K, fmt, seed=0, out="fp16"):
    import torch
    rng = np.random.default_rng(seed + M * 13 + N + K)
    W_bits = _weights(rng, N, K)
    X = rng.standard_normal((M, K)).astype(np.float32)
    sal = rng.choice(K, size=max(1, round(0.01 * K)), replace=False)
    X[:, sal] *= 20
    X_bits = X.astype(np.float16).view(np.uint16)
    codes, bs, gs = _oracle_quant(W_bits, fmt)
    What = oracle.nvfp4_dequant(codes, bs, gs) if fmt == "nvfp4" else oracle.mxfp4_dequant(codes, bs)
    Y_ref = oracle.gemm_f32(oracle.f16_to_f32(X_bits), What.astype(np.float32))
    qw = dev(oracle.pack_device(codes).view(np.int32))
    bsd = dev(np.ascontiguousarray(bs.T))
    tsd = None if gs is None else dev(np.array([gs], np.float32))
    tdt = {"fp16": torch.float16, "fp32": torch.float32}[out]
    Y = w4.w4a16_fp4_gemm(dev_bits(X_bits, torch.float16), qw, bsd, tsd, fmt, out_dtype=tdt)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    return check_y(to_f64(Y), Y_ref, out)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 33, 64])
def test_fp4_gemm_decode_token_counts(fmt, M):
    skip_without_gpu()
    _gemm_case(M, 256, 1024, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(16, 64), (144, 320), (400, 4096), (4096, 128)])
def test_fp4_gemm_ragged_shapes(fmt, N, K):
    skip_without_gpu()
    _gemm_case(2, N, K, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(65, 256, 1024), (200, 384, 2048), (512, 144, 320)])
def test_fp4_gemm_prefill(fmt, M, N, K):
    """M > 64: the tcgen05 kernel on weights decoded with their block scale."""
    skip_without_gpu()
    _gemm_case(M, N, K, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp4_gemm_fp32_output(fmt):
    skip_without_gpu()
    _gemm_case(4, 512, 2048, fmt, out="fp32")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layer", [0, 2, 3])
def test_fp4_llama7b_layers_m1(fmt, layer):
    """Full-size 7B projections at M = 1: the GPU quantiser packs the weights (its parity
    is tested above); the oracle quantises independently and computes sampled rows."""
    skip_without_gpu()
    import torch
    wl = workloads.workload(2)
    li = workloads.make_layer(wl, layer, M=1)
    W_bits = li.W.view(np.uint16)
    Wd = dev_bits(W_bits, torch.float16)
    qw, bsd, tsd = w4.w4_fp4_quantize_pack(Wd, fmt)
    Y = w4.w4a16_fp4_gemm(dev_bits(li.X, torch.float16), qw, bsd, tsd, fmt)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    rng = np.random.default_rng(layer)
    ns = np.unique(np.concatenate([[0, li.N - 1], rng.integers(0, li.N, 256)]))
    if fmt == "nvfp4":
        # the tensor scale depends on the whole tensor: take the oracle's on all rows
        codes, bs, gs = oracle.nvfp4_quantize(W_bits)
        What = oracle.nvfp4_dequant(codes[ns], bs[ns], gs)
    else:
        codes, es = oracle.mxfp4_quantize(W_bits[ns])
        What = oracle.mxfp4_dequant(codes, es)
    Y_ref = oracle.gemm_f32(oracle.f16_to_f32(li.X), What.astype(np.float32))
    check_y(to_f64(Y)[:, ns], Y_ref, "fp16")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layer", [0, 1])
def test_fp4_llama8b_prefill_m4096(fmt, layer):
    """The 8B-shaped prefill projections at M = 4096 with fp16 activations (the FP4 path
    takes fp16), oracle on sampled output rows and columns."""
    skip_without_gpu()
    import torch
    wl = workloads.workload(4)
    L = wl.layers[layer]
    M = 4096
    W_bits = workloads.gen_weights(L.N, L.K, 0, 4, layer).view(np.uint16)
    X_bits = workloads.gen_acts(M, L.K, 0, 4, layer, "fp16")
    qw, bsd, tsd = w4.w4_fp4_quantize_pack(dev_bits(W_bits, torch.float16), fmt)
    Y = w4.w4a16_fp4_gemm(dev_bits(X_bits, torch.float16), qw, bsd, tsd, fmt, out_dtype=torch.float32)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    rng = np.random.default_rng(layer + 40)
    ms = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 24)]))
    ns = np.unique(np.concatenate([[0, L.N - 1], rng.integers(0, L.N, 128)]))
    if fmt == "nvfp4":
        codes, bs, gs = oracle.nvfp4_quantize(W_bits)
        What = oracle.nvfp4_dequant(codes[ns], bs[ns], gs)
    else:
        codes, es = oracle.mxfp4_quantize(W_bits[ns])
        What = oracle.mxfp4_dequant(codes, es)
    Y_ref = oracle.gemm_f32(oracle.f16_to_f32(X_bits), What.astype(np.float32), rows=ms)
    check_y(to_f64(Y)[np.ix_(ms, ns)], Y_ref, "fp32")


def test_fp4_gemm_refuses_bf16_activations():
    skip_without_gpu()
    import torch
    X = torch.zeros(1, 128, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(256 * 128 // 8, dtype=torch.int32, device="cuda")
    bs = torch.zeros(8, 256, dtype=torch.uint8, device="cuda")
    ts = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_fp4_gemm(X, qw, bs, ts, "nvfp4")
    assert e.value.status == w4.W4_ERR_UNSUPPORTED
