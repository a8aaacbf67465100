"""Pins of the oracle's AWQ scale search (CPU): the candidates reduce to plain RTN when
every channel has the same activation magnitude, salient channels make a positive
exponent win (the premise of "Quantization Paradigms for Edge Inference: AWQ, GPTQ, and
FP8 Matrix Cores", sec. 3), columns whose mean magnitudes are powers of two give the
candidates in closed form, and each loss equals the squared error summed by explicit
loops on a tiny layer."""
import numpy as np

import oracle


def layer(rng, M, N, K, salient=True):
    x = rng.standard_normal((M, K)).astype(np.float32)
    if salient:
        x[:, rng.choice(K, size=max(1, K // 100), replace=False)] *= 20
    W = (rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)).astype(np.float16)
    return x.astype(np.float16).view(np.uint16), W.view(np.uint16)


def test_equal_magnitudes_give_unit_scales_and_plain_rtn():
    rng = np.random.default_rng(0)
    M, N, K, g = 8, 32, 256, 64
    X = (rng.choice([-1.0, 1.0], size=(M, K)) * 0.5).astype(np.float16).view(np.uint16)
    _, W = layer(rng, M, N, K)
    best, losses, s = oracle.awq_search(W, X, g, symmetric=False, n_grid=5)
    assert best == 0
    assert np.all(s == np.float32(1))
    assert np.all(losses == losses[0])
    # the loss of s = 1: plain RTN, X' = X
    q, sc, zr = oracle.quantize_weights(W, None, g, False)
    Xf = oracle.f16_to_f32(X)
    Yref = oracle.gemm_f32(Xf, oracle.f16_to_f32(W)).astype(np.float64)
    Yq = oracle.gemm_f32(Xf, oracle.dequant(q, sc, zr, g)).astype(np.float64)
    assert losses[0] == ((Yref - Yq) ** 2).sum()


def test_salient_channels_make_a_positive_exponent_win():
    rng = np.random.default_rng(1)
    X, W = layer(rng, 16, 64, 512)
    best, losses, s = oracle.awq_search(W, X, 128, symmetric=False, n_grid=10)
    assert best > 0
    assert losses[best] < 0.9 * losses[0]
    assert not np.all(s == np.float32(1))


def test_losses_match_explicit_sums_on_a_tiny_layer():
    rng = np.random.default_rng(2)
    M, N, K, g, n_grid = 3, 16, 64, 32, 3
    X, W = layer(rng, M, N, K)
    best, losses, _ = oracle.awq_search(W, X, g, symmetric=True, n_grid=n_grid)
    Xf = oracle.f16_to_f32(X).astype(np.float64)
    Wf = oracle.f16_to_f32(W).astype(np.float64)
    m = [sum(abs(Xf[i, k]) for i in range(M)) / M for k in range(K)]
    lm = [np.log(v) for v in m]
    mu = sum(lm) / K
    for j in range(n_grid):
        s = np.array([np.exp((j / n_grid) * (v - mu)) for v in lm], np.float32)
        q, sc, _ = oracle.quantize_weights(W, s, g, True)
        scf = oracle.f16_to_f32(sc).astype(np.float64)
        tot = 0.0
        for i in range(M):
            for n in range(N):
                ref = sum(Xf[i, k] * Wf[n, k] for k in range(K))
                yq = 0.0
                for k in range(K):
                    xp = oracle.f16_to_f32(oracle.f32_to_f16(np.float32(Xf[i, k]) * (np.float32(1) / s[k]))).item()
                    yq += xp * (int(q[n, k]) - 8) * scf[k // g, n]
                tot += (ref - yq) ** 2
        assert abs(losses[j] - tot) <= 1e-5 * tot
    assert best == int(np.argmin(losses))


def test_power_of_two_magnitudes_give_closed_form_candidates():
    """Column k has mean magnitude exactly 2^e[k] (e even, mean 0), half the columns as
    +-2^e and half as +-2^(e-1) / +-3*2^(e-1) (so max / mean differs between columns).  The
    geometric mean of m^a is then 1, and the candidate a = 1/2 is exactly s = 2^(e/2):
    its loss must be that of quantising with this closed-form s, and a = 0 that of plain
    RTN."""
    rng = np.random.default_rng(3)
    M, N, K, g = 8, 32, 256, 64
    half = rng.choice([-4, -2, 0, 2, 4], size=K // 2)
    e = rng.permutation(np.concatenate([half, -half]))
    mag = np.ldexp(np.ones((M, K)), np.broadcast_to(e, (M, K)))
    two_level = np.arange(K) % 2 == 1
    mult = np.where(np.arange(M)[:, None] % 2 == 0, 0.5, 1.5)
    mag = np.where(two_level[None, :], mag * mult, mag)
    X = (rng.choice([-1.0, 1.0], size=(M, K)) * mag).astype(np.float16)
    assert np.array_equal(np.abs(X.astype(np.float64)).mean(axis=0), np.ldexp(1.0, e))
    X = X.view(np.uint16)
    _, W = layer(rng, M, N, K, salient=False)
    _, losses, _ = oracle.awq_search(W, X, g, symmetric=False, n_grid=2)

    def loss_with(s):
        q, sc, zr = oracle.quantize_weights(W, s, g, False)
        Xf = oracle.f16_to_f32(X)
        # X / s is exact here (powers of two), so no rounding of X' enters
        Xp = Xf if s is None else Xf / s
        Yref = oracle.gemm_f32(Xf, oracle.f16_to_f32(W)).astype(np.float64)
        Yq = oracle.gemm_f32(Xp, oracle.dequant(q, sc, zr, g)).astype(np.float64)
        return ((Yref - Yq) ** 2).sum()

    assert losses[0] == loss_with(None)
    assert losses[1] == loss_with(np.ldexp(np.float32(1), e // 2).astype(np.float32))
