"""GPU parity of w4_quantize_pack: bit-exact against the CPU oracle (packed words in the
device layout and in canonical order, fp16 scales, fp16 zero points)."""
import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from bit_weight_only_w4_b200 import workloads
from tests.gpu_util import act_order, dev, dev_bits, host_bits, host_u32, skip_without_gpu

pytestmark = pytest.mark.gpu


def run_and_compare(W_bits, s, g, sym, g_idx, bf16_w=False):
    import torch
    N, K = W_bits.shape
    Wd = dev_bits(W_bits, torch.bfloat16 if bf16_w else torch.float16)
    qw, sc, zr = w4.w4_quantize_pack(Wd, dev(s), g, sym, dev(g_idx))
    can = w4.w4_unpack_canonical(qw, N, K)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    q, sc_ref, zr_ref = oracle.quantize_weights(W_bits, s, g, sym, g_idx, is_bf16=bf16_w)
    assert np.array_equal(host_bits(sc), sc_ref)
    if sym:
        assert zr is None
    else:
        assert np.array_equal(host_bits(zr), zr_ref)
    assert np.array_equal(host_u32(qw), oracle.pack_device(q))
    assert np.array_equal(host_u32(can), oracle.pack_canonical(q))


@pytest.mark.parametrize("N,K,g,sym,gidx,bf16_w,with_s", [
    (16, 64, 32, False, False, False, True),      # one tile
    (48, 192, 64, False, False, False, True),     # ragged: 3 tiles x 3 atoms
    (32, 256, 256, True, False, False, False),    # per-channel, symmetric
    (64, 512, 128, True, True, False, True),      # act-order
    (64, 512, 32, False, True, False, True),      # act-order, asymmetric, g=32
    (32, 384, 128, False, False, True, True),     # bf16 weights
    (16, 64, 64, False, False, False, False),
])
def test_quantize_small(N, K, g, sym, gidx, bf16_w, with_s):
    skip_without_gpu()
    rng = np.random.default_rng(N * 1000 + K + g)
    Wf = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    if bf16_w:
        W_bits = oracle.f32_to_bf16(Wf)
    else:
        W_bits = Wf.astype(np.float16).view(np.uint16)
    s = np.exp(rng.uniform(-1.5, 1.5, K)).astype(np.float32) if with_s else None
    g_idx = act_order(rng, K, g) if gidx else None
    run_and_compare(W_bits, s, g, sym, g_idx, bf16_w)


def test_quantize_degenerate_groups():
    skip_without_gpu()
    # all-zero rows, constant groups, ties exactly half-way between grid points
    N, K, g = 32, 128, 32
    W = np.zeros((N, K), np.float32)
    W[1, :32] = 0.25
    sc = 2.0 ** -7
    W[2] = ((np.arange(K) % 16) - 7.5) * sc
    W[3, ::2] = 1e-7
    run_and_compare(W.astype(np.float16).view(np.uint16), None, g, False, None)
    run_and_compare(W.astype(np.float16).view(np.uint16), None, g, True, None)


@pytest.mark.parametrize("config_id,layer,g", [(1, 0, 128), (2, 3, 128), (5, 0, 32), (5, 0, 4096)])
def test_quantize_config_layers(config_id, layer, g):
    """Full-size layers of the measured workloads (whole matrix compared)."""
    skip_without_gpu()
    wl = workloads.workload(config_id)
    li = workloads.make_layer(wl, layer, M=1, group_size=g)
    run_and_compare(li.W.view(np.uint16), li.s, li.group_size, li.symmetric, li.g_idx)


def test_quantize_70b_gate_up_sampled_bands():
    """The largest layer (57344 x 8192): GPU over the whole matrix, oracle on sampled
    128-row bands (first, last and seeded random ones); a band's packed words are one
    contiguous run of the device layout."""
    skip_without_gpu()
    import torch
    wl = workloads.workload(3)
    li = workloads.make_layer(wl, 2, M=1)
    N, K, g = li.N, li.K, li.group_size
    qw, sc, zr = w4.w4_quantize_pack(dev_bits(li.W.view(np.uint16), torch.float16), dev(li.s), g)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    bands = sorted(set([0, N // 128 - 1] + rng.integers(0, N // 128, 4).tolist()))
    words = K // 64 * 128 * 8
    qw_h, sc_h, zr_h = host_u32(qw), host_bits(sc), host_bits(zr)
    for b in bands:
        rows = slice(128 * b, 128 * b + 128)
        q, s_ref, z_ref = oracle.quantize_weights(li.W.view(np.uint16)[rows], li.s, g)
        assert np.array_equal(qw_h[b * words:(b + 1) * words], oracle.pack_device(q))
        assert np.array_equal(sc_h[:, rows], s_ref)
        assert np.array_equal(zr_h[:, rows], z_ref)
