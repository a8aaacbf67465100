"""Helpers shared by the GPU parity tests: move seeded host arrays to the device, run the
library through its binding, and compare with the CPU oracle."""
import numpy as np
import pytest

import oracle

RELL2_TOL = 1e-3      # relative L2 error bound on Y (fp16 / fp32 outputs)
MAXABS_TOL = 2e-2     # max-abs error bound on Y (fp16 / fp32 outputs)


def torch_mod():
    import torch
    return torch


def dev_bits(bits, dtype):
    """uint16 bit patterns (numpy) -> CUDA tensor of the given 16-bit float dtype."""
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).cuda()


def dev(a):
    torch = torch_mod()
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t):
    """CUDA fp16/bf16 tensor -> numpy uint16 bit patterns."""
    torch = torch_mod()
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def host_u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def to_f64(t):
    torch = torch_mod()
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float32 \
        else t.detach().cpu().numpy().astype(np.float64)


def random_layer(rng, M, N, K, act="fp16", salient=True):
    """Small seeded layer in the shape of the measured workloads (X ~ N(0,1) with 1%
    salient channels x20, W ~ N(0, 0.02), s from |X| of a calibration batch)."""
    x = rng.standard_normal((M, K)).astype(np.float32)
    cal = rng.standard_normal((64, K)).astype(np.float32)
    if salient:
        sal = rng.choice(K, size=max(1, round(0.01 * K)), replace=False)
        x[:, sal] *= 20
        cal[:, sal] *= 20
    s = np.sqrt(np.maximum(np.abs(cal).mean(0), 1e-6)).astype(np.float64)
    s = (s / np.exp(np.log(s).mean())).astype(np.float32)
    s_inv = (np.float32(1) / s).astype(np.float32)
    W = (rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)).astype(np.float16)
    if act == "fp16":
        X = x.astype(np.float16).view(np.uint16)
    else:
        X = oracle.f32_to_bf16(x)
    return X, W.view(np.uint16), s, s_inv


def act_order(rng, K, g):
    perm = rng.permutation(K)
    pos = np.empty(K, np.int64)
    pos[perm] = np.arange(K)
    return (pos // g).astype(np.int32)


def check_y(Y_gpu, Y_ref, out_dtype, tol_rel=RELL2_TOL, tol_abs=MAXABS_TOL, absprod=None,
            act_round=0.0, K=None):
    """Y within the stated tolerance of the oracle's fp32 result (fp16 / fp32 outputs).

    bf16 outputs: bf16 rounding alone exceeds that tolerance, so each element must lie
    within one bf16 ulp of the oracle value plus the error the fp32 path may carry --
    act_round * sum_k |X'[m,k] What[n,k]| when X' is rounded to the activation type
    before the MMA, and (K+2) 2^-24 of the same sum for fp32 accumulation."""
    Y_gpu = np.asarray(Y_gpu, np.float64)
    Y_ref = np.asarray(Y_ref, np.float64)
    assert Y_gpu.shape == Y_ref.shape
    assert np.all(np.isfinite(Y_gpu))
    err = Y_gpu - Y_ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(Y_ref), 1e-30)
    mx = np.abs(err).max() if err.size else 0.0
    if out_dtype == "bf16":
        mag = np.maximum(np.abs(Y_ref), 2.0 ** -126)
        ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
        allow = ulp.copy()
        if absprod is not None:
            allow += (act_round + (K + 2) * 2.0 ** -24) * np.asarray(absprod, np.float64)
        bad = np.abs(err) > allow * (1 + 1e-9)
        assert not bad.any(), (int(bad.sum()), Y_gpu[bad][:4], Y_ref[bad][:4])
    else:
        assert rel <= tol_rel, f"relL2 {rel:.3e} > {tol_rel}"
        assert mx <= tol_abs, f"max abs {mx:.3e} > {tol_abs}"
    return rel, mx


def skip_without_gpu():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
