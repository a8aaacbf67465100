"""Pins for the oracle's packing, its reference product and the measurement arithmetic.

  * Canonical / device packing: hand-derived words (tests/golden/pack_words.txt) and
    round trips on random codes (edgesiliconlab.com article on AWQ vs GPTQ, "Kernel
    Execution: Marlin vs. ExLlamaV2 INT4 GEMM Micro-Architecture", item 3).
  * Reference product: brute force against exact sums of the fp32 products with the
    recursive-summation error bound, a closed-form special case (all weights one -> row
    sums), numpy fp64 matmul on mid shapes, and the fp64 companion.
  * Roofline and byte accounting against the pages' worked examples
    (tests/golden/roofline_worked_example.txt).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_weight_only_w4_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pattern(name, N, K):
    r = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    if name == "col":
        q = (k % 16 + 4 * ((r % 16) // 8)) % 16
    elif name == "row":
        q = np.broadcast_to(r % 16, (N, K))
    elif name == "tile":
        q = 4 * (r // 16) + k // 64
    elif name == "band":
        q = (r // 16 + 3 * (k // 64)) % 16
    else:
        raise KeyError(name)
    return np.ascontiguousarray(q, dtype=np.uint8)


def _golden_pack_lines():
    out = []
    for line in open(os.path.join(GOLDEN, "pack_words.txt")):
        if line.startswith("#") or not line.strip():
            continue
        lhs, rhs = line.split("=")
        out.append((lhs.split(), int(rhs.strip(), 16)))
    return out


@pytest.mark.parametrize("case", range(len(_golden_pack_lines())))
def test_pack_golden_words(case):
    fields, word = _golden_pack_lines()[case]
    if fields[0] == "canonical":
        q = np.array([int(v) for v in fields[1:]], np.uint8).reshape(1, -1)
        assert oracle.pack_canonical(q)[0, 0] == word
    else:
        _, pat, N, K, idx = fields
        qd = oracle.pack_device(_pattern(pat, int(N), int(K)))
        assert qd[int(idx)] == word, hex(int(qd[int(idx)]))


@pytest.mark.parametrize("N,K", [(16, 64), (48, 192), (32, 4096), (160, 128), (272, 320)])
def test_pack_round_trips(N, K):
    rng = np.random.default_rng(N + K)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    qc = oracle.pack_canonical(q)
    assert qc.shape == (N, K // 8)
    assert np.array_equal(oracle.unpack_canonical(qc, K), q)
    qd = oracle.pack_device(q)
    assert qd.size == N * K // 8
    assert np.array_equal(oracle.unpack_device(qd, N, K), q)
    # device packing is a permutation of the canonical nibbles: same multiset per tile
    assert sorted(_nibbles(qd)) == sorted(_nibbles(qc.reshape(-1)))


def _nibbles(words):
    w = np.asarray(words, np.uint32)
    return np.concatenate([(w >> (4 * i)) & 0xF for i in range(8)]).tolist()


def test_pack_all_byte_pairs():
    # every pair of adjacent codes (all 256 x 256 combinations of two bytes of codes)
    a = np.arange(65536)
    q = np.stack([(a >> (4 * i)) & 0xF for i in range(4)] * 2, axis=1).astype(np.uint8)
    qc = oracle.pack_canonical(q)
    assert np.array_equal(oracle.unpack_canonical(qc, 8), q)
    assert np.array_equal(qc[:, 0] & 0xFFFF, a.astype(np.uint32))


def test_device_pack_rejects_untiled_shapes():
    with pytest.raises(ValueError):
        oracle.pack_device(np.zeros((8, 64), np.uint8))
    with pytest.raises(ValueError):
        oracle.pack_device(np.zeros((16, 32), np.uint8))


# ---------------------------------------------------------------- reference product
def _exact_dot(x, w):
    return sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x, w)), Fraction(0))


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 8, 64), (8, 3, 8), (1, 64, 64)])
def test_gemm_brute_force_bound(M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    Xp = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    What = (rng.integers(-15, 16, size=(N, K)) * rng.choice([2**-8, 2**-6], (N, 1))) \
        .astype(np.float32)
    Y = oracle.gemm_f32(Xp, What)
    u = 2.0 ** -24
    for m in range(M):
        for n in range(N):
            exact = _exact_dot(Xp[m], What[n])
            absum = sum(abs(float(a) * float(b)) for a, b in zip(Xp[m], What[n]))
            bound = (K + 1) * u * absum * (1 + 1e-6)
            assert abs(Fraction(float(Y[m, n])) - exact) <= Fraction(bound) + Fraction(1, 10**30)


def test_gemm_all_ones_gives_row_sums():
    # q - z = 1 and sc = 1 everywhere: What == 1, so Y[m,n] = sum_k X'[m,k]
    M, N, K = 4, 16, 128
    rng = np.random.default_rng(2)
    X = rng.standard_normal((M, K)).astype(np.float16).view(np.uint16)
    q = np.full((N, K), 9, np.uint8)
    scales = np.full((K // 64, N), 0x3C00, np.uint16)   # 1.0
    zeros = np.full((K // 64, N), 0x4000, np.uint16)    # 2.0 ... then q - z = 7
    What = oracle.dequant(q, scales, zeros, 64)
    assert np.all(What == 7.0)
    zeros[:] = 0x4800                                   # 8.0 -> q - z = 1
    What = oracle.dequant(q, scales, zeros, 64)
    assert np.all(What == 1.0)
    Y = oracle.reference_y(X, None, q, scales, zeros, 64)
    x = X.view(np.float16).astype(np.float64)
    for m in range(M):
        exact = math.fsum(x[m])
        assert np.allclose(Y[m], exact, rtol=0, atol=K * 2**-24 * np.abs(x[m]).sum())


def test_gemm_matches_numpy_fp64_and_companion():
    rng = np.random.default_rng(9)
    M, N, K = 7, 96, 1024
    Xp = rng.standard_normal((M, K)).astype(np.float32)
    What = (rng.integers(-15, 16, (N, K)) * 0.01).astype(np.float32)
    Y32 = oracle.gemm_f32(Xp, What)
    Y64 = oracle.gemm_f64(Xp, What)
    ref = Xp.astype(np.float64) @ What.astype(np.float64).T
    assert np.linalg.norm(Y64 - ref) <= 1e-12 * np.linalg.norm(ref)
    assert np.linalg.norm(Y32 - ref) <= 1e-5 * np.linalg.norm(ref)
    rows = np.array([6, 0, 3], np.int64)
    assert np.array_equal(oracle.gemm_f32(Xp, What, rows), Y32[rows])


def test_dequant_uses_group_index():
    # swapping the groups of two channels through g_idx swaps which scale they use
    N, K, g = 16, 64, 32
    q = np.full((N, K), 10, np.uint8)
    scales = np.stack([np.full(N, 0x3C00), np.full(N, 0x4000)]).astype(np.uint16)  # 1, 2
    zeros = np.full((2, N), 0x4400, np.uint16)                                      # 4
    g_idx = (np.arange(K) // g).astype(np.int32)
    g_idx[[0, 40]] = g_idx[[40, 0]]
    What = oracle.dequant(q, scales, zeros, g, g_idx)
    assert What[0, 0] == 12.0 and What[0, 40] == 6.0 and What[0, 1] == 6.0


# ---------------------------------------------------------------- measurement arithmetic
def _golden_roofline():
    vals = {}
    for line in open(os.path.join(GOLDEN, "roofline_worked_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        t = line.split()
        vals[t[0]] = t[1:]
    return vals


def test_roofline_worked_example():
    v = _golden_roofline()
    bw = float(v["bandwidth_gbs"][0])
    fp16 = workloads.roofline_tokens_per_s(bw, float(v["fp16_model_gb"][0]))
    awq = workloads.roofline_tokens_per_s(bw, float(v["awq4_model_gb"][0]))
    assert fp16 == pytest.approx(float(v["fp16_model_gb"][2]), abs=1e-9)
    assert math.floor(awq * 10) / 10 == pytest.approx(float(v["awq4_model_gb"][2]))


def test_footprints_match_pages():
    v = _golden_roofline()
    p70 = float(v["params_70b"][0])
    p7 = float(v["params_7b"][0])
    # fp16: 2 bytes per weight; packed INT4: half a byte per weight (codes only)
    assert 2 * p70 / 1e9 == float(v["params_70b"][2])
    # a square-ish stand-in with exactly p weights: codes = p / 2 bytes
    N, K = 7000, 1_000_000
    codes_only = workloads.effective_weight_bytes(N, K, K, True, False) - 2 * N
    assert codes_only / 1e9 == float(v["params_7b"][2]) == p7 / 2 / 1e9
    N, K = 70000, 1_000_000
    codes_only = workloads.effective_weight_bytes(N, K, K, True, False) - 2 * N
    assert codes_only / 1e9 == float(v["params_70b"][4])


def test_effective_bytes_metadata_terms():
    # asymmetric g128: 0.5 B/weight + 4 B per (group, column); symmetric + g_idx: 2 B + 4K
    assert workloads.effective_weight_bytes(4096, 4096, 128, False, False) == \
        4096 * 4096 // 2 + 4 * 32 * 4096
    assert workloads.effective_weight_bytes(11008, 4096, 128, True, True) == \
        11008 * 4096 // 2 + 2 * 32 * 11008 + 4 * 4096
