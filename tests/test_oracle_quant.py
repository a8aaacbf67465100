"""Pins for the oracle's AWQ transform, group-wise RTN quantisation and dequantisation.

Pins (none retypes the oracle's formulas):
  * AWQ identity ("Quantization Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix
    Cores", sec. 3, eq. 1): with power-of-two s the transformed product is bit-identical.
  * On-grid closed form: weights built as (q - z) * sc with sc a power of two and every
    group spanning codes 0 and 15 must come back as exactly those q, z, sc (fp16 and
    bf16 weights).
  * bf16 operands of the transform are read as bf16 (the format's top-half definition).
  * Brute force of round-to-nearest-even over all 16 codes.
  * Range properties of the scale / zero point; reconstruction error <= sc/2.
  * A hand-worked group (tests/golden/quant_hand_example.txt).
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16bits(x):
    return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------- AWQ identity (eq. 1)
@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (5, 16, 128), (3, 24, 96)])
def test_awq_identity_bit_exact_with_power_of_two_scales(M, N, K):
    rng = np.random.default_rng(M * 100 + N)
    X = f16bits(rng.standard_normal((M, K)))
    W = f16bits(rng.standard_normal((N, K)) * 0.02)
    s = (2.0 ** rng.integers(-3, 4, size=K)).astype(np.float32)
    s_inv = (np.float32(1) / s).astype(np.float32)
    Wp = oracle.awq_scale_weights(W, s)
    Xp = oracle.awq_scale_acts(X, s_inv)
    W0 = oracle.awq_scale_weights(W, None)
    X0 = oracle.awq_scale_acts(X, None)
    # the transform really scaled something, along k
    assert not np.array_equal(Wp, W0)
    assert np.array_equal(Wp[:, s == 1], W0[:, s == 1])
    Y_scaled = oracle.gemm_f32(Xp, Wp)
    Y_plain = oracle.gemm_f32(X0, W0)
    assert np.array_equal(Y_scaled.view(np.uint32), Y_plain.view(np.uint32))


def test_awq_identity_random_scales_fp64():
    rng = np.random.default_rng(5)
    M, N, K = 4, 16, 256
    X = f16bits(rng.standard_normal((M, K)))
    W = f16bits(rng.standard_normal((N, K)) * 0.02)
    s = np.exp(rng.uniform(-2, 2, K)).astype(np.float32)
    Xp = oracle.awq_scale_acts(X, (np.float32(1) / s).astype(np.float32)).astype(np.float64)
    Wp = oracle.awq_scale_weights(W, s).astype(np.float64)
    X0 = X.view(np.float16).astype(np.float64)
    W0 = W.view(np.float16).astype(np.float64)
    Y1 = Xp @ Wp.T
    Y0 = X0 @ W0.T
    # two fp32 roundings per product: relative error of order 2^-23
    assert np.linalg.norm(Y1 - Y0) <= 4e-7 * np.linalg.norm(Y0) + 1e-12


# ---------------------------------------------------------------- on-grid closed form
def _on_grid(N, K, g, symmetric, rng, g_idx=None):
    G = K // g
    sc = (2.0 ** rng.integers(-9, -5, size=(G, N))).astype(np.float32)
    z = np.full((G, N), 8) if symmetric else rng.integers(1, 15, size=(G, N))
    lo = 1 if symmetric else 0
    q = rng.integers(lo, 16, size=(N, K))
    grp = (np.arange(K) // g) if g_idx is None else g_idx
    # force every group to contain both extreme codes
    for gg in range(G):
        ks = np.nonzero(grp == gg)[0]
        q[:, ks[0]] = lo
        q[:, ks[1]] = 15
    W = ((q - z[grp, :].T) * sc[grp, :].T).astype(np.float32)
    assert np.array_equal(W.astype(np.float16).astype(np.float32), W)  # exact in fp16
    return f16bits(W), q.astype(np.uint8), sc, z


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("g,act_order", [(32, False), (64, False), (128, True), (256, False)])
def test_on_grid_weights_recovered_exactly(symmetric, g, act_order):
    rng = np.random.default_rng(g + 3 * symmetric)
    N, K = 16, 512
    g_idx = None
    if act_order:
        perm = rng.permutation(K)
        pos = np.empty(K, np.int64)
        pos[perm] = np.arange(K)
        g_idx = (pos // g).astype(np.int32)
    W, q_true, sc_true, z_true = _on_grid(N, K, g, symmetric, rng, g_idx)
    q, scales, zeros = oracle.quantize_weights(W, None, g, symmetric, g_idx)
    assert np.array_equal(q, q_true)
    assert np.array_equal(oracle.f16_to_f32(scales), sc_true)
    if symmetric:
        assert zeros is None
    else:
        assert np.array_equal(oracle.f16_to_f32(zeros), z_true.astype(np.float32))
    # dequantisation of the on-grid case reproduces the weights exactly
    What = oracle.dequant(q, scales, zeros, g, g_idx)
    assert np.array_equal(What, W.view(np.float16).astype(np.float32))


def bf16_exact(W32):
    """bf16 bit patterns of fp32 values that bf16 holds exactly: the upper 16 bits."""
    W32 = np.ascontiguousarray(W32, np.float32)
    assert np.all((W32.view(np.uint32) & 0xFFFF) == 0)
    return (W32.view(np.uint32) >> 16).astype(np.uint16)


def bf16_decode(b):
    """bf16 bit patterns -> fp32 by the format's definition (the bits are fp32's top half)."""
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("symmetric", [False, True])
def test_on_grid_bf16_weights_recovered_exactly(symmetric):
    """bf16 weights: (q - z) * 2^e needs at most 4 significant bits, so the on-grid weights
    are exact in bf16 too and must come back as exactly q, z, sc."""
    rng = np.random.default_rng(71 + symmetric)
    N, K, g = 16, 256, 64
    W16, q_true, sc_true, z_true = _on_grid(N, K, g, symmetric, rng)
    Wb = bf16_exact(W16.view(np.float16).astype(np.float32))
    q, scales, zeros = oracle.quantize_weights(Wb, None, g, symmetric, is_bf16=True)
    assert np.array_equal(q, q_true)
    assert np.array_equal(oracle.f16_to_f32(scales), sc_true)
    if not symmetric:
        assert np.array_equal(oracle.f16_to_f32(zeros), z_true.astype(np.float32))


def test_awq_transform_reads_bf16_operands_as_bf16():
    """The transform of bf16 operands decodes them as bf16: without s it returns the decoded
    values, and with power-of-two s it scales them exactly (no rounding can occur)."""
    rng = np.random.default_rng(72)
    M, N, K = 3, 8, 64
    Xb = bf16_exact(oracle.bf16_to_f32(oracle.f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))))
    Wb = bf16_exact(oracle.bf16_to_f32(oracle.f32_to_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))))
    s = (2.0 ** rng.integers(-3, 4, size=K)).astype(np.float32)
    s_inv = (np.float32(1) / s).astype(np.float32)
    assert np.array_equal(oracle.awq_scale_acts(Xb, None, True), bf16_decode(Xb))
    assert np.array_equal(oracle.awq_scale_weights(Wb, None, True), bf16_decode(Wb))
    assert np.array_equal(oracle.awq_scale_acts(Xb, s_inv, True), bf16_decode(Xb) * s_inv)
    assert np.array_equal(oracle.awq_scale_weights(Wb, s, True), bf16_decode(Wb) * s)


@pytest.mark.parametrize("symmetric", [False, True])
def test_exact_ties_round_to_even(symmetric):
    # weights exactly half-way between two grid points: W'/sc = j + 0.5 exactly, so
    # rint must return the even integer -- independent of the (often odd) zero point
    rng = np.random.default_rng(31 + symmetric)
    N, K, g = 16, 64, 32
    G = K // g
    sc = 2.0 ** -7
    W = np.zeros((N, K))
    expect = np.zeros((N, K), bool)
    for n in range(N):
        for gg in range(G):
            ks = np.arange(gg * g, (gg + 1) * g)
            if symmetric:
                z = 8
                W[n, ks[0]], W[n, ks[1]] = -7 * sc, 7 * sc          # absmax = 7 sc
                lo, hi = -7, 6
            else:
                z = int(rng.integers(1, 15))
                W[n, ks[0]], W[n, ks[1]] = -z * sc, (15 - z) * sc   # range = 15 sc
                lo, hi = -z, 14 - z
            j = rng.integers(lo, hi + 1, size=g - 2)
            W[n, ks[2:]] = (j + 0.5) * sc
            expect[n, ks[2:]] = True
    Wb = f16bits(W)
    assert np.array_equal(Wb.view(np.float16).astype(np.float64), W)
    q, scales, zeros = oracle.quantize_weights(Wb, None, g, symmetric)
    assert np.all(oracle.f16_to_f32(scales) == sc)
    z = np.full((G, N), 8.0) if symmetric else oracle.f16_to_f32(zeros)
    zk = z[np.arange(K) // g, :].T
    d = q.astype(np.float64) - zk           # the rounded integer rint(W'/sc)
    half = W / sc
    assert np.all(np.abs(d[expect] - half[expect]) == 0.5)
    assert np.all(d[expect] % 2 == 0)


def test_hand_worked_group():
    vals = {}
    for line in open(os.path.join(GOLDEN, "quant_hand_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *rest = line.split()
        vals[key] = rest
    W = np.array([int(v, 16) for v in vals["weights_fp16_bits"]], np.uint16).reshape(1, -1)
    g = int(vals["group_size"][0])
    q, scales, zeros = oracle.quantize_weights(W, None, g)
    assert scales[0, 0] == int(vals["scale_fp16_bits"][0], 16)
    assert zeros[0, 0] == int(vals["zero_fp16_bits"][0], 16)
    assert q[0].tolist() == [int(v) for v in vals["codes"]]


# ---------------------------------------------------------------- brute force RTN
@pytest.mark.parametrize("symmetric", [False, True])
def test_rtn_brute_force_and_bounds(symmetric):
    rng = np.random.default_rng(11 + symmetric)
    N, K, g = 8, 256, 32
    W = f16bits(rng.standard_normal((N, K)) * 0.02)
    s = np.exp(rng.uniform(-1, 1, K)).astype(np.float32)
    Wp = oracle.awq_scale_weights(W, s)
    q, scales, zeros = oracle.quantize(Wp, g, symmetric)
    sc = oracle.f16_to_f32(scales)              # [G,N]
    z = np.full_like(sc, 8.0) if symmetric else oracle.f16_to_f32(zeros)
    assert q.min() >= 0 and q.max() <= 15
    assert np.all((z >= 0) & (z <= 15) & (z == np.round(z)))
    grp = np.arange(K) // g
    codes = np.arange(16, dtype=np.float64)
    for n in range(N):
        for k in range(K):
            s_nk = np.float32(sc[grp[k], n])
            z_nk = float(z[grp[k], n])
            t = float(np.float32(Wp[n, k]) / s_nk)      # IEEE fp32 quotient
            # nearest integer to t over the whole integer line, ties to the even integer
            d = np.abs(t - (codes - z_nk))
            cand = codes[d == d.min()]
            if cand.size > 1:
                cand = cand[((cand - z_nk) % 2) == 0]
            best = float(cand[0])
            # the nearest code (ties to the even integer) is the rounded, clamped value
            assert q[n, k] == best, (n, k, t, z_nk, q[n, k], best)
            if -0.5 <= t + z_nk <= 15.5:
                # not clamped: reconstruction error at most half a step
                assert abs((q[n, k] - z_nk) * s_nk - Wp[n, k]) <= s_nk / 2 * (1 + 2**-20)


@pytest.mark.parametrize("symmetric", [False, True])
def test_scale_covers_group_range(symmetric):
    rng = np.random.default_rng(21 + symmetric)
    N, K, g = 16, 512, 128
    W = f16bits(rng.standard_normal((N, K)) * 0.02)
    Wp = oracle.awq_scale_weights(W, None)
    q, scales, zeros = oracle.quantize(Wp, g, symmetric)
    sc = oracle.f16_to_f32(scales).astype(np.float64)
    z = np.full_like(sc, 8.0) if symmetric else oracle.f16_to_f32(zeros).astype(np.float64)
    Wg = Wp.reshape(N, K // g, g).astype(np.float64)
    mn, mx = Wg.min(-1).T, Wg.max(-1).T   # [G,N]
    am = np.abs(Wg).max(-1).T
    rel = 2.0 ** -11                       # fp16 rounding of the scale
    if symmetric:
        # 7 steps cover the largest magnitude
        assert np.all(np.abs(7 * sc - am) <= rel * am + 1e-12)
    else:
        # 15 steps span the group's range and the grid brackets both ends
        assert np.all(np.abs(15 * sc - (mx - mn)) <= rel * (mx - mn) + 1e-12)
        assert np.all(-z * sc <= mn + sc / 2 + 1e-12)
        assert np.all((15 - z) * sc >= mx - sc / 2 - 1e-12)


def test_degenerate_groups_get_minimum_scale():
    # an all-zero group and a constant group: scale floors at the smallest fp16 normal
    W = np.zeros((16, 64), np.float32)
    W[1, :32] = 0.25
    q, scales, zeros = oracle.quantize(W, 32, False)
    assert scales[0, 0] == 0x0400 and scales[0, 1] == 0x0400
    assert np.all(q[0] == q[0, 0])
    # the zero point is the integer 0, stored as +0 (never the fp16 pattern of -0)
    assert zeros[0, 0] == 0x0000 and zeros[0, 1] == 0x0000


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 100), np.float32), 32)
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 64), np.float32), 32, True, np.full(64, 5, np.int32))
