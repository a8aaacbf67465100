"""GPU parity of w4a16_gemm_chain (a list of decode GEMMs in one persistent launch)
against the CPU oracle run layer by layer.

The oracle chain rounds every layer's output to the output type, as the GPU stores it,
and feeds the next layer the same slice the GPU layer reads.  It also rounds each layer's
X' = X s^-1 to the activation type before the product, as the kernels do: through a deep
chain the per-layer X' rounding (about 1.4e-4 relative L2 a layer) otherwise accumulates
like a random walk (about 1e-3 after 40 layers) and would hide what the chain test is
for.  fp16 chains are then held to the stated bound (relative L2 1e-3, max-abs 2e-2): the
chains differ only where the GPU's fp32 summation order moves a value across an fp16
rounding boundary (a 1-ulp difference on a small fraction of elements), and such
differences pass through later layers at about their own relative size.  bf16 outputs are
held to one bf16 ulp of the oracle plus the fp32 path's error bound.
"""
import numpy as np
import pytest

import oracle
import bit_weight_only_w4_b200 as w4
from bit_weight_only_w4_b200 import workloads
from tests.gpu_util import check_y, dev, dev_bits, random_layer, skip_without_gpu, to_f64

pytestmark = pytest.mark.gpu


def _round(y32, bf16):
    return oracle.f32_to_bf16(y32) if bf16 else oracle.f32_to_f16(y32)


def _oracle_layer(Xb, s_inv, q, sc, zr, g, bf16):
    """One layer of the oracle chain: X' = X s^-1 in fp32, rounded to the activation type
    (as the kernels round it), then the dequantised weights and the fp32 product."""
    Xp = oracle.awq_scale_acts(Xb, s_inv, bf16)
    Xp = oracle.bf16_to_f32(oracle.f32_to_bf16(Xp)) if bf16 else oracle.f16_to_f32(oracle.f32_to_f16(Xp))
    return oracle.gemm_f32(Xp, oracle.dequant(q, sc, zr, g))


def _build(M, specs, seed, act="fp16", g=128):
    """specs: list of (K, N, source layer or -1, first column).  Returns the device layer
    list, the oracle's per-layer outputs (fp32 and rounded bits) and the host inputs."""
    import torch
    bf16 = act == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float16
    rng = np.random.default_rng(seed)
    K0 = specs[0][0]
    X0, _, _, _ = random_layer(rng, M, 16, K0, act)
    layers, ref32, refbits, host = [], [], [], []
    X0d = dev_bits(X0, tdt)
    ys = []
    for j, (K, N, src, c0) in enumerate(specs):
        _, W, s, s_inv = random_layer(rng, 1, N, K, act)
        s_inv = workloads.chain_s_inv(s_inv)
        q, sc, zr = oracle.quantize_weights(W, s, g)
        Y = torch.full((M, N), float("nan"), dtype=tdt, device="cuda")
        ys.append(Y)
        Xd = (X0d if src < 0 else ys[src])[:, c0:c0 + K]
        Xb = (X0 if src < 0 else refbits[src])[:, c0:c0 + K]
        y = _oracle_layer(np.ascontiguousarray(Xb), s_inv, q, sc, zr, g, bf16)
        ref32.append(y)
        refbits.append(_round(y, bf16))
        host.append({"Xbits": np.ascontiguousarray(Xb), "q": q, "sc": sc, "zr": zr, "s_inv": s_inv})
        layers.append({"X": Xd, "qweight": dev(oracle.pack_device(q).view(np.int32)),
                       "scales": dev_bits(sc, torch.float16), "zeros": dev_bits(zr, torch.float16),
                       "s_inv": dev(s_inv), "Y": Y, "group_size": g})
    return layers, ref32, host


def _run(layers, workspace=None):
    import torch
    w4.w4a16_gemm_chain(layers, workspace=workspace)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    return [to_f64(d["Y"]) for d in layers]


# every layer reads its predecessor's output (at columns 0 and 256)
SMALL = [(512, 1536, -1, 0), (512, 512, 0, 0), (512, 1024, 1, 0), (768, 512, 2, 256),
         (512, 768, 3, 0)]
# layer 1 reads layer 0 at column 64 (a slice that starts inside a 16-byte chunk of the
# row) and layer 2 reads layer 0 (not its predecessor); layers 3 and 4 read their
# predecessors
MIXED = [(512, 1536, -1, 0), (512, 512, 0, 64), (512, 1024, 0, 512), (768, 512, 2, 256),
         (512, 768, 3, 0)]


@pytest.mark.parametrize("M,specs", [(1, "small"), (2, "small"), (3, "small"), (8, "small"),
                                     (1, "mixed"), (8, "mixed")])
def test_chain_small_matches_oracle_chain(M, specs):
    skip_without_gpu()
    layers, ref32, _ = _build(M, SMALL if specs == "small" else MIXED, seed=M)
    for _ in range(2):                         # twice: the counter is left at zero
        ys = _run(layers)
        for y, r in zip(ys, ref32):
            check_y(y, r, "fp16")


def test_chain_longer_than_one_launch_in_a_graph():
    """40 layers: two launches (32 + 8).  Layers 31 -> 32 -> 33 read their predecessor
    across the launch boundary (as do 1 and 2 at the start); the others read the block
    input, so no dependency path is longer than four layers (each layer adds about 1.5e-4
    of relative error against the oracle -- the fp32 fold of the biased codes and the fp16
    output -- and a 40-deep path would add up to the stated bound by itself).  Captured
    in a CUDA graph and replayed."""
    skip_without_gpu()
    import torch
    chained = {1, 2, 31, 32, 33}
    specs = [(256, 256, -1, 0)] + [(256, 256, j - 1 if j in chained else -1, 0) for j in range(1, 40)]
    M = 2
    layers, ref32, _ = _build(M, specs, seed=7)
    _run(layers)                               # eager once
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            w4.w4a16_gemm_chain(layers)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        for d in layers:
            d["Y"].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        w4.w4_check_device_error()
        for d, r in zip(layers, ref32):
            check_y(to_f64(d["Y"]), r, "fp16")


@pytest.mark.parametrize("act,specs,M", [("fp16", "small", 3), ("fp16", "mixed", 3), ("bf16", "small", 2),
                                         ("bf16", "mixed", 1)])
def test_chain_matches_separate_gemm_calls(act, specs, M):
    """Each layer of the chain computes exactly what w4a16_gemm computes for the same
    input: fed the chain's own intermediate outputs, the separate calls agree bit for bit
    (same kernel arithmetic, same deterministic split-K order)."""
    skip_without_gpu()
    import torch
    layers, _, _ = _build(M, SMALL if specs == "small" else MIXED, seed=99, act=act)
    ys = _run(layers)
    for j, d in enumerate(layers):
        X = d["X"].contiguous()
        Y = w4.w4a16_gemm(X, d["qweight"], d["scales"], d["zeros"], 128, s_inv=d["s_inv"])
        torch.cuda.synchronize()
        assert np.array_equal(to_f64(Y), ys[j]), f"layer {j}"


def test_chain_llama7b_block():
    """One block of the 7B-shaped decode step at full size (M = 1): qkv -> o -> gate_up ->
    down, each projection fed from the previous output as the step's stand-in defines."""
    skip_without_gpu()
    import torch
    wl = workloads.workload(2)
    M = 1
    li0 = workloads.make_layer(wl, 0, M=M)
    X0 = li0.X
    ys, layers, refbits = [], [], []
    for j, L in enumerate(wl.layers):
        li = workloads.make_layer(wl, j, M=M)
        s_inv = workloads.chain_s_inv(li.s_inv)
        W_bits = li.W.view(np.uint16)
        q, sc, zr = oracle.quantize_weights(W_bits, li.s, li.group_size)
        src, c0 = workloads.CHAIN_SOURCE[j]
        Xb = X0 if src < 0 else refbits[src][:, c0:c0 + L.K]
        y = _oracle_layer(np.ascontiguousarray(Xb), s_inv, q, sc, zr, li.group_size, False)
        refbits.append(oracle.f32_to_f16(y))
        Y = torch.full((M, L.N), float("nan"), dtype=torch.float16, device="cuda")
        Xd = dev_bits(X0, torch.float16) if src < 0 else ys[src][:, c0:c0 + L.K]
        ys.append(Y)
        layers.append({"X": Xd, "qweight": dev(oracle.pack_device(q).view(np.int32)),
                       "scales": dev_bits(sc, torch.float16), "zeros": dev_bits(zr, torch.float16),
                       "s_inv": dev(s_inv), "Y": Y, "group_size": li.group_size, "ref": y})
    out = _run([{k: v for k, v in d.items() if k != "ref"} for d in layers])
    for y, d in zip(out, layers):
        rel, mx = check_y(y, d["ref"], "fp16")
        assert np.abs(d["ref"]).max() < 64.0   # the stand-in gains keep values O(1)


def test_chain_bf16():
    """bf16 activations and outputs.  The layers read slices of the block input (exact on
    both sides), so each output is held to the per-element bf16 rule: one bf16 ulp of the
    oracle's fp32 value plus the error the fp32 path may carry (X' rounded to bf16 before
    the MMA: 2^-8 of sum|X' What|; fp32 accumulation: (K+2) 2^-24 of it).  Propagation
    through a chain is covered by the fp16 tests."""
    skip_without_gpu()
    M = 2
    specs = [(512, 1024, -1, 0), (512, 512, -1, 0), (256, 512, -1, 256)]
    layers, ref32, host = _build(M, specs, seed=5, act="bf16")
    ys = _run(layers)
    for y, r, h in zip(ys, ref32, host):
        Xp = oracle.awq_scale_acts(h["Xbits"], h["s_inv"], True).astype(np.float64)
        What = oracle.dequant(h["q"], h["sc"], h["zr"], 128).astype(np.float64)
        check_y(y, r, "bf16", absprod=np.abs(Xp) @ np.abs(What).T, act_round=2.0 ** -8,
                K=What.shape[1])


def test_chain_refuses_what_it_does_not_run():
    skip_without_gpu()
    import torch
    M = 9                                      # more than one token tile
    X = torch.zeros(M, 256, dtype=torch.float16, device="cuda")
    qw = torch.zeros(256 * 256 // 8, dtype=torch.int32, device="cuda")
    sc = torch.ones(2, 256, dtype=torch.float16, device="cuda")
    Y = torch.empty(M, 256, dtype=torch.float16, device="cuda")
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemm_chain([{"X": X, "qweight": qw, "scales": sc, "zeros": sc, "Y": Y}])
    assert e.value.status == w4.W4_ERR_UNSUPPORTED
    # two group modes in one list
    X1 = X[:1]
    Y1 = torch.empty(1, 256, dtype=torch.float16, device="cuda")
    sc32 = torch.ones(8, 256, dtype=torch.float16, device="cuda")
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemm_chain([{"X": X1, "qweight": qw, "scales": sc, "zeros": sc, "Y": Y1},
                             {"X": Y1, "qweight": qw, "scales": sc32, "zeros": sc32, "Y": Y1,
                              "group_size": 32}])
    assert e.value.status == w4.W4_ERR_UNSUPPORTED
