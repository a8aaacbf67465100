"""Pins of the oracle's block-scaled 4-bit floating point (NVFP4, MXFP4; "Production
Quantization: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4", section "MXFP4 / NVFP4": a
scale factor per block of weights).  The element and scale formats are the published
definitions, read in w4_oracle.c; the pins are:
  * E2M1: the format's table of 16 values; hand-derived round-to-nearest-even at every
    midpoint; nearest-value property over a dense grid; saturation beyond 6.
  * E4M3: all 256 codes against torch.float8_e4m3fn; rounding against torch's cast over
    random and midpoint values inside the range; saturation to 448 beyond it.
  * NVFP4 / MXFP4 block quantisation: tensors built on the grid (elements times
    representable block scales, a tensor scale that is a power of two, every block
    holding its largest element) come back as exactly those codes and scales;
    reconstruction error bounded by the block scale on random data, each element a
    nearest point of the grid of its stored block scale; blocks independent.
"""
import numpy as np
import pytest
import torch

import oracle

# E2M1 magnitudes by code 0..7 (sign in bit 3): the format's value table
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_table():
    for c in range(16):
        v = oracle.e2m1_to_f32(c)
        mag = E2M1[c & 7]
        assert abs(v) == mag and (np.signbit(v) == bool(c & 8))


@pytest.mark.parametrize("x,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),   # midpoints: even mantissa
    (0.2, 0), (0.3, 1), (1.3, 3), (2.6, 5), (4.9, 6), (5.1, 7), (6.0, 7),
    (7.0, 7), (1e6, 7),                                                         # saturation
    (-0.75, 10), (-5.0, 14), (-100.0, 15),
])
def test_e2m1_encode_hand_derived(x, code):
    assert oracle.f32_to_e2m1(x) == code


def test_e2m1_encode_is_nearest():
    xs = np.linspace(-7.0, 7.0, 2801).astype(np.float32)
    mags = np.array(E2M1)
    for x in xs:
        v = oracle.e2m1_to_f32(oracle.f32_to_e2m1(float(x)))
        best = np.min(np.abs(abs(float(x)) - mags))
        assert abs(abs(v) - abs(float(x))) == best
        assert v == 0.0 or np.sign(v) == np.sign(x)


def test_e4m3_decode_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for b in range(256):
        v = oracle.e4m3_to_f32(b)
        if np.isnan(ref[b]):
            assert np.isnan(v)
        else:
            assert v == ref[b] and np.signbit(v) == np.signbit(ref[b])


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.uniform(-460, 460, 4000),
        rng.standard_normal(4000) * 0.05,
        np.ldexp(rng.uniform(-1, 1, 2000), rng.integers(-12, 9, 2000)),
    ]).astype(np.float32)
    # exact midpoints between neighbouring codes (ties to even)
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    for x in (464.0, 480.0, 1e4, 3e38):
        assert oracle.f32_to_e4m3(x) == 0x7E
        assert oracle.f32_to_e4m3(-x) == 0xFE


def _e4m3_values():
    return torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def test_nvfp4_on_grid_recovered_exactly():
    rng = np.random.default_rng(1)
    R, K = 6, 128
    gs = np.float32(2.0 ** -10)
    e4 = _e4m3_values()
    normal = np.flatnonzero(e4 >= 0.125)             # block scales well inside fp16's range
    sb = rng.choice(normal, size=(R, K // 16)).astype(np.uint8)
    sb[0, 0] = 0x7E                                   # one block at 448: amax = 6 * 448 * gs
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    codes[:, ::16] = rng.choice([7, 15], size=(R, K // 16))   # every block holds +-6
    dec = np.array([E2M1[c & 7] * (-1 if c & 8 else 1) for c in codes.ravel()]).reshape(R, K)
    scale = e4[sb].repeat(16, axis=1).astype(np.float64) * float(gs)
    W = (dec * scale).astype(np.float16)
    assert np.array_equal(W.astype(np.float64), dec * scale)        # exact in fp16
    q, bs, g = oracle.nvfp4_quantize(W.view(np.uint16))
    assert g == gs
    assert np.array_equal(bs, sb)
    # codes equal, except that +0 and -0 may be written either way by the fp16 cast
    same = (q == codes) | (((q & 7) == 0) & ((codes & 7) == 0))
    assert same.all()
    assert np.array_equal(oracle.nvfp4_dequant(q, bs, g), W.astype(np.float64))


def test_nvfp4_error_bound_and_block_independence():
    rng = np.random.default_rng(2)
    R, K = 8, 256
    W = (rng.standard_normal((R, K)) * 0.05).astype(np.float16)
    W[0, 0] = 1.0                                      # fixes the tensor scale
    q, bs, g = oracle.nvfp4_quantize(W.view(np.uint16))
    What = oracle.nvfp4_dequant(q, bs, g)
    sd = np.array([[oracle.e4m3_to_f32(b) for b in row] for row in bs]).repeat(16, axis=1) * float(g)
    err = np.abs(W.astype(np.float64) - What)
    # half the widest E2M1 gap (1, between 4 and 6) plus the block scale's rounding
    assert np.all(err <= 1.5 * sd + 1e-30)
    # every element is a nearest point of the grid its STORED block scale defines; the
    # decision is taken on the fp32 quotient w / (scale * gs), so a near-tie may go either
    # way within that quotient's rounding (a few 2^-24 of |w|)
    absw = np.abs(W.astype(np.float64))
    grid = np.abs(absw[:, :, None] - np.array(E2M1)[None, None, :] * sd[:, :, None])
    assert np.all(err <= grid.min(axis=2) + 2.0 ** -21 * absw + 1e-30)
    # a change inside one block leaves every other block's codes and scales alone
    W2 = W.copy()
    W2[3, 32:48] *= np.float16(0.5)
    q2, bs2, g2 = oracle.nvfp4_quantize(W2.view(np.uint16))
    assert g2 == g
    mask = np.ones((R, K), bool)
    mask[3, 32:48] = False
    assert np.array_equal(q2[mask], q[mask])
    bmask = np.ones(bs.shape, bool)
    bmask[3, 2] = False
    assert np.array_equal(bs2[bmask], bs[bmask])


def test_mxfp4_on_grid_recovered_exactly():
    rng = np.random.default_rng(3)
    R, K = 4, 128
    e = rng.integers(-8, 4, size=(R, K // 32))
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    codes[:, ::32] = rng.choice([6, 7, 14, 15], size=(R, K // 32))   # block max 4 or 6 (x 2^e)
    dec = np.array([E2M1[c & 7] * (-1 if c & 8 else 1) for c in codes.ravel()]).reshape(R, K)
    W = np.ldexp(dec, e.repeat(32, axis=1)).astype(np.float16)
    assert np.array_equal(W.astype(np.float64), np.ldexp(dec, e.repeat(32, axis=1)))
    q, es = oracle.mxfp4_quantize(W.view(np.uint16))
    assert np.array_equal(es.astype(np.int64) - 127, e)
    same = (q == codes) | (((q & 7) == 0) & ((codes & 7) == 0))
    assert same.all()
    assert np.array_equal(oracle.mxfp4_dequant(q, es), W.astype(np.float64))


def test_mxfp4_scale_is_the_blocks_leading_power_of_two_over_four():
    # a block whose largest magnitude is 1.0 gets scale 2^-2 and the element 1.0 -> code 4.0
    W = np.zeros((1, 32), np.float16)
    W[0, 5] = 1.0
    W[0, 9] = -0.3
    q, es = oracle.mxfp4_quantize(W.view(np.uint16))
    assert int(es[0, 0]) - 127 == -2
    assert oracle.e2m1_to_f32(q[0, 5]) == 4.0
    # -0.3 / 0.25 = -1.2 -> nearest E2M1 is -1.0
    assert oracle.e2m1_to_f32(q[0, 9]) == -1.0


def test_block_sizes_are_enforced():
    with pytest.raises(ValueError):
        oracle.nvfp4_quantize(np.zeros((1, 24), np.float16).view(np.uint16))
    with pytest.raises(ValueError):
        oracle.mxfp4_quantize(np.zeros((1, 48), np.float16).view(np.uint16))
