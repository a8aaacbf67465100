"""Pins for the oracle's IEEE-754 binary16 / bfloat16 converters.

The converters are written from the format definitions; here they are checked against
library routines (numpy float16 casts, torch bfloat16 casts), exhaustively where the
domain is 2^16 and on random plus constructed halfway values otherwise.
"""
import numpy as np
import pytest
import torch

import oracle


def _same_bits_or_both_nan(a_bits, b_bits, is_bf16):
    a = np.asarray(a_bits, np.uint16)
    b = np.asarray(b_bits, np.uint16)
    if is_bf16:
        nan_a = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
        nan_b = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    else:
        nan_a = ((a & 0x7C00) == 0x7C00) & ((a & 0x3FF) != 0)
        nan_b = ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)
    ok = (a == b) | (nan_a & nan_b)
    return ok


def test_f16_to_f32_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def _f32_probe_values(rng, n):
    # random bit patterns over the whole float32 range
    raw = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32).view(np.float32)
    # values in and around the fp16 range
    mid = (rng.standard_normal(n) * rng.choice([1e-8, 1e-5, 1e-3, 1, 1e3, 6e4, 7e4], n)) \
        .astype(np.float32)
    return np.concatenate([raw, mid])


def _f16_halfway_values():
    # exact midpoints between adjacent finite fp16 values (and +/- the next float32 around
    # them): the ties-to-even cases
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)  # exact: needs at most 12 significant bits
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    v = np.concatenate([mid, up, dn, [65504.0, 65519.996, 65520.0, 65536.0, 1e-8, 2.0**-25,
                                      2.0**-24, 3 * 2.0**-26]]).astype(np.float32)
    return np.concatenate([v, -v])


def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(123)
    v = np.concatenate([_f32_probe_values(rng, 400_000), _f16_halfway_values()])
    ours = oracle.f32_to_f16(v)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    ok = _same_bits_or_both_nan(ours, ref, is_bf16=False)
    assert ok.all(), (v[~ok][:8], ours[~ok][:8], ref[~ok][:8])


def test_bf16_to_f32_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(7)
    v = _f32_probe_values(rng, 400_000)
    # bf16 halfway cases: low 16 bits exactly 0x8000 on random high halves
    hi = rng.integers(0, 2**16, size=50_000, dtype=np.uint64).astype(np.uint32)
    half = ((hi << 16) | 0x8000).astype(np.uint32).view(np.float32)
    v = np.concatenate([v, half, np.float32([3.3895314e38, 3.4028235e38, 1e-45, -0.0])])
    ours = oracle.f32_to_bf16(v)
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ok = _same_bits_or_both_nan(ours, ref, is_bf16=True)
    assert ok.all(), (v[~ok][:8], ours[~ok][:8], ref[~ok][:8])


@pytest.mark.parametrize("x", [0.0, 1.0, -2.5, 65504.0, 2.0**-14, 2.0**-24])
def test_f16_roundtrip_scalars(x):
    b = oracle.lib().oracle_f32_to_f16(x)
    assert oracle.lib().oracle_f16_to_f32(b) == x
