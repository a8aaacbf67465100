"""GPU parity of act-order weights with contiguous groups: w4_actorder_perm, w4_quantize_pack
with perm and w4a16_gemm with perm, against the oracle's g_idx quantisation and product.

- perm must equal a stable sort of g_idx (bit-exact), and map every group onto one
  contiguous run of group_size columns;
- the packed codes, scales and zero points must equal the oracle's g_idx quantisation with
  the columns taken in perm order (bit-exact: the groups and their members are the same);
- Y must lie within the GEMM tolerance of the oracle's g_idx product (the same sum, taken
  in another order), for the decode and the prefill kernels.
"""
import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from tests.gpu_util import (act_order, check_y, dev, dev_bits, host_bits, host_u32, random_layer,
                            skip_without_gpu, to_f64)

pytestmark = pytest.mark.gpu


def gpu_perm(g_idx, g):
    import torch
    perm = w4.w4_actorder_perm(dev(g_idx), g)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), w4.lib().w4_check_device_error()


@pytest.mark.parametrize("K,g", [(1024, 32), (1024, 128), (11008, 128), (4096, 4096), (352, 32)])
def test_perm_is_a_stable_sort_of_g_idx(K, g):
    skip_without_gpu()
    rng = np.random.default_rng(K + g)
    g_idx = act_order(rng, K, g)
    perm, st = gpu_perm(g_idx, g)
    assert st == w4.W4_OK
    assert np.array_equal(perm, np.argsort(g_idx, kind="stable"))
    # every group is one contiguous run, its channels ascending
    assert np.array_equal(g_idx[perm], np.arange(K) // g)
    assert np.all(np.diff(perm.reshape(-1, g), axis=1) > 0)


def test_perm_reports_uneven_groups_and_bad_entries():
    skip_without_gpu()
    K, g = 512, 64
    rng = np.random.default_rng(5)
    g_idx = act_order(rng, K, g)
    uneven = g_idx.copy()
    uneven[np.flatnonzero(uneven == 0)[0]] = 1          # group 0 one short, group 1 one over
    assert gpu_perm(uneven, g)[1] == w4.W4_ERR_DEVICE_ARG
    out_of_range = g_idx.copy()
    out_of_range[7] = K // g
    assert gpu_perm(out_of_range, g)[1] == w4.W4_ERR_DEVICE_ARG
    assert gpu_perm(g_idx, g)[1] == w4.W4_OK            # the error word was cleared


@pytest.mark.parametrize("N,K,g,sym,with_s", [
    (64, 512, 128, True, True),
    (48, 1024, 32, False, True),      # ragged band (3 tiles), asymmetric, g = 32
    (32, 256, 64, True, False),
])
def test_pack_with_perm_is_gidx_quantisation_in_perm_order(N, K, g, sym, with_s):
    skip_without_gpu()
    import torch
    rng = np.random.default_rng(N * 7 + K + g)
    W = (rng.standard_normal((N, K)).astype(np.float32) * 0.02).astype(np.float16).view(np.uint16)
    s = np.exp(rng.uniform(-1.5, 1.5, K)).astype(np.float32) if with_s else None
    g_idx = act_order(rng, K, g)
    perm = np.argsort(g_idx, kind="stable").astype(np.int32)
    qw, sc, zr = w4.w4_quantize_pack(dev_bits(W, torch.float16), dev(s), g, sym, perm=dev(perm))
    can = w4.w4_unpack_canonical(qw, N, K)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    q, sc_ref, zr_ref = oracle.quantize_weights(W, s, g, sym, g_idx)
    # the groups are the same, so the scales and zero points are too
    assert np.array_equal(host_bits(sc), sc_ref)
    if sym:
        assert zr is None
    else:
        assert np.array_equal(host_bits(zr), zr_ref)
    # column k' of the packed matrix is channel perm[k']
    assert np.array_equal(host_u32(can), oracle.pack_canonical(q[:, perm]))
    assert np.array_equal(host_u32(qw), oracle.pack_device(q[:, perm]))


def perm_case(M, N, K, g, sym, act="fp16", out="fp16", use_s=True, seed=0):
    import torch
    rng = np.random.default_rng(seed + M * 131 + N + K + g)
    X, W, s, s_inv = random_layer(rng, M, N, K, act)
    g_idx = act_order(rng, K, g)
    q, scales, zeros = oracle.quantize_weights(W, s, g, sym, g_idx)
    perm = np.argsort(g_idx, kind="stable").astype(np.int32)
    qd = oracle.pack_device(q[:, perm])                  # the layout w4_quantize_pack(perm=) writes
    tdt = {"fp16": torch.float16, "bf16": torch.bfloat16, "fp32": torch.float32}
    s_call = s_inv if use_s else None
    Y = w4.w4a16_gemm(dev_bits(X, tdt[act]), dev(qd.view(np.int32)), dev_bits(scales, torch.float16),
                      None if zeros is None else dev_bits(zeros, torch.float16), g, s_inv=dev(s_call),
                      out_dtype=tdt[out], perm=dev(perm))
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    Y_ref = oracle.reference_y(X, s_call, q, scales, zeros, g, g_idx, x_is_bf16=(act == "bf16"))
    kw = {}
    if out == "bf16":
        Xp = oracle.awq_scale_acts(X, s_call, act == "bf16").astype(np.float64)
        What = oracle.dequant(q, scales, zeros, g, g_idx).astype(np.float64)
        kw["absprod"] = np.abs(Xp) @ np.abs(What).T
        kw["act_round"] = 0.0 if s_call is None else (2.0 ** -8 if act == "bf16" else 2.0 ** -11)
        kw["K"] = K
    return check_y(to_f64(Y), Y_ref, out, **kw)


@pytest.mark.parametrize("M", [1, 5, 16, 33, 64])
@pytest.mark.parametrize("g", [32, 128])
def test_gemm_perm_decode(M, g):
    skip_without_gpu()
    perm_case(M, 256, 1024, g, sym=True)


def test_gemm_perm_asymmetric_bf16_no_s():
    skip_without_gpu()
    perm_case(3, 144, 512, 64, sym=False, act="bf16", out="bf16", use_s=False)


@pytest.mark.parametrize("M,g", [(200, 128), (130, 32)])
def test_gemm_perm_prefill(M, g):
    skip_without_gpu()
    perm_case(M, 384, 1024, g, sym=True)


def test_gemm_perm_full_size_workload():
    """The act-order workload's shape (4096 -> 11008, symmetric, g = 128) at M = 1, with
    the permutation computed on the GPU and the weights packed by the GPU quantiser."""
    skip_without_gpu()
    import torch
    from bit_weight_only_w4_b200 import workloads
    wl = workloads.workload(5)
    li = workloads.make_layer(wl, 0, M=1, group_size=128)
    perm = w4.w4_actorder_perm(dev(li.g_idx), 128)
    Wd = dev_bits(li.W.view(np.uint16), torch.float16)
    s = dev(li.s) if li.s is not None else None
    qw, sc, _ = w4.w4_quantize_pack(Wd, s, 128, True, perm=perm)
    X = dev_bits(li.X, torch.float16)
    si = dev(li.s_inv) if li.s_inv is not None else None
    Y = w4.w4a16_gemm(X, qw, sc, None, 128, s_inv=si, perm=perm)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    # sampled output columns against the oracle (quantised with g_idx on the host)
    cols = np.unique(np.concatenate([[0, li.N - 1], np.random.default_rng(3).choice(li.N, 62, replace=False)]))
    q, scales, _ = oracle.quantize_weights(li.W.view(np.uint16)[cols], li.s, 128, True, li.g_idx)
    Y_ref = oracle.reference_y(li.X, li.s_inv, q, scales, None, 128, li.g_idx)
    check_y(to_f64(Y)[:, cols], Y_ref, "fp16")
