"""Seeded synthetic workloads for the W4A16 path (inputs only -- no quantisation math).

Both the CUDA path and the CPU oracle consume the arrays built here; this module holds
none of the method's arithmetic (no scaling of weights, no rounding to INT4, no packing).

Shapes stand in for the linear layers of the 7B / 8B / 70B models that the pages discuss
("Quantization Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix Cores", sec. 1
footprints; "Production Quantization" lesson, AWQ / GPTQ-Marlin figures at 7B).  No
dataset or trained weight is involved: values are drawn from a documented generator.

Generator: numpy PCG64 seeded by SeedSequence([seed, config_id, layer_key, tensor_id]).
  X  ~ N(0,1) (float32 draws), with round(0.01 K) salient input channels (chosen by seed,
       without replacement) multiplied by 20, rounded to the activation dtype (RNE).
  W  = fp16(0.02 * N(0,1)) (float32 draws), shape [N, K] (out x in).
  s  : stand-in for the AWQ scale search -- s_k = (mean_m |Xcal[m,k]|)^0.5 over a
       128-row calibration batch drawn like X (same salient set), mean floored at 1e-6,
       normalised to geometric mean 1 in fp64, then rounded to fp32; s_inv = 1/s in fp32.
  g_idx (act-order): a seeded permutation perm of [0,K); channel k sits at position
       pos[k] (pos[perm[i]] = i) and belongs to group pos[k] // g, so every group has
       exactly g channels.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

CALIB_ROWS = 128
SALIENT_FRACTION = 0.01
SALIENT_GAIN = 20.0
W_STD = 0.02

# tensor ids for the seed sequence
_T_SALIENT, _T_X, _T_CAL, _T_W, _T_PERM = 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Layer:
    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    """One of the five measured workloads."""
    config_id: int
    name: str
    layers: Tuple[Layer, ...]
    Ms: Tuple[int, ...]
    act_dtype: str = "fp16"          # "fp16" or "bf16"
    group_sizes: Tuple[int, ...] = (128,)
    symmetric: bool = False
    act_order: bool = False
    prescaled_acts: bool = False     # X arrives already multiplied by s^-1 (s_inv not passed)
    note: str = ""


WORKLOADS: Tuple[Workload, ...] = (
    Workload(1, "single_4096", (Layer("linear", 4096, 4096),), (1,),
             note="single linear layer, M=1, K=N=4096, asymmetric g128, AWQ s"),
    Workload(2, "llama7b_decode",
             (Layer("qkv", 4096, 12288), Layer("o", 4096, 4096),
              Layer("gate_up", 4096, 22016), Layer("down", 11008, 4096)),
             (1, 2, 4, 8, 16),
             note="Llama-7B-shaped decode GEMV sweep, asymmetric g128, AWQ s"),
    Workload(3, "llama70b_decode",
             (Layer("qkv", 8192, 10240), Layer("o", 8192, 8192),
              Layer("gate_up", 8192, 57344), Layer("down", 28672, 8192)),
             (1, 8, 32, 64),
             note="70B-shaped decode and small-batch layers, asymmetric g128, AWQ s"),
    Workload(4, "llama8b_prefill",
             (Layer("up", 4096, 14336), Layer("down", 14336, 4096)),
             (512, 2048, 4096, 8192), act_dtype="bf16", prescaled_acts=True,
             note="8B-shaped prefill GEMMs, bf16 activations pre-scaled by s^-1, asymmetric g128"),
    Workload(5, "gptq_actorder", (Layer("linear", 4096, 11008),), (1, 16, 1024),
             group_sizes=(32, 64, 128, 4096), symmetric=True, act_order=True,
             note="GPTQ-style symmetric INT4 (implicit zero 8), act-order g_idx"),
)


def workload(config_id: int) -> Workload:
    for w in WORKLOADS:
        if w.config_id == config_id:
            return w
    raise KeyError(config_id)


def rng_for(seed: int, config_id: int, layer_key: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([seed, config_id, layer_key, tensor_id])))


def salient_channels(K: int, seed: int, config_id: int, layer_key: int) -> np.ndarray:
    count = int(round(SALIENT_FRACTION * K))
    r = rng_for(seed, config_id, layer_key, _T_SALIENT)
    return np.sort(r.choice(K, size=count, replace=False))


def _to_act_dtype(x32: np.ndarray, act_dtype: str) -> np.ndarray:
    """Round fp32 values to the activation dtype (RNE); returns uint16 bit patterns."""
    if act_dtype == "fp16":
        return x32.astype(np.float16).view(np.uint16)
    if act_dtype == "bf16":
        import torch
        return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).view(torch.int16) \
            .numpy().view(np.uint16)
    raise ValueError(act_dtype)


def gen_acts(M: int, K: int, seed: int, config_id: int, layer_key: int,
             act_dtype: str = "fp16", tensor_id: int = _T_X) -> np.ndarray:
    """X [M,K] as uint16 bit patterns of fp16 / bf16."""
    r = rng_for(seed, config_id, layer_key, tensor_id)
    x = r.standard_normal((M, K), dtype=np.float32)
    sal = salient_channels(K, seed, config_id, layer_key)
    x[:, sal] *= np.float32(SALIENT_GAIN)
    return _to_act_dtype(x, act_dtype)


def gen_weights(N: int, K: int, seed: int, config_id: int, layer_key: int,
                chunk_rows: int = 4096) -> np.ndarray:
    """W [N,K] fp16 (as numpy float16)."""
    r = rng_for(seed, config_id, layer_key, _T_W)
    W = np.empty((N, K), np.float16)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        W[r0:r1] = (r.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(W_STD)) \
            .astype(np.float16)
    return W


def awq_scales(K: int, seed: int, config_id: int, layer_key: int,
               act_dtype: str = "fp16") -> Tuple[np.ndarray, np.ndarray]:
    """Closed-form stand-in for the AWQ search: s_k = mean|Xcal_k|^0.5, geometric mean 1."""
    cal_bits = gen_acts(CALIB_ROWS, K, seed, config_id, layer_key, act_dtype, tensor_id=_T_CAL)
    if act_dtype == "fp16":
        cal = cal_bits.view(np.float16).astype(np.float64)
    else:
        cal = (cal_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mean_abs = np.maximum(np.abs(cal).mean(axis=0), 1e-6)
    s = np.sqrt(mean_abs)
    s = s / np.exp(np.log(s).mean())
    s32 = s.astype(np.float32)
    s_inv = (np.float32(1.0) / s32).astype(np.float32)
    return s32, s_inv


def act_order_gidx(K: int, group_size: int, seed: int, config_id: int, layer_key: int) -> np.ndarray:
    perm = rng_for(seed, config_id, layer_key, _T_PERM).permutation(K)
    pos = np.empty(K, np.int64)
    pos[perm] = np.arange(K)
    return (pos // group_size).astype(np.int32)


@dataclass
class LayerInputs:
    K: int
    N: int
    M: int
    act_dtype: str
    X: np.ndarray                 # uint16 bits [M,K]; already scaled by s^-1 if prescaled
    W: np.ndarray                 # float16 [N,K]
    s: np.ndarray                 # float32 [K]
    s_inv: Optional[np.ndarray]   # float32 [K], None when X is pre-scaled
    group_size: int
    symmetric: bool
    g_idx: Optional[np.ndarray]   # int32 [K] or None


def make_layer(wl: Workload, layer_index: int, M: int, group_size: Optional[int] = None,
               seed: int = 0, with_weights: bool = True) -> LayerInputs:
    layer = wl.layers[layer_index]
    g = group_size if group_size is not None else wl.group_sizes[0]
    key = layer_index
    s, s_inv = awq_scales(layer.K, seed, wl.config_id, key, wl.act_dtype)
    X = gen_acts(M, layer.K, seed, wl.config_id, key, wl.act_dtype)
    if wl.prescaled_acts:
        # activations as the previous op would emit them with s^-1 already absorbed
        if wl.act_dtype == "fp16":
            x32 = X.view(np.float16).astype(np.float32)
        else:
            x32 = (X.astype(np.uint32) << 16).view(np.float32)
        X = _to_act_dtype((x32 * s_inv[None, :]).astype(np.float32), wl.act_dtype)
        s_call = None
    else:
        s_call = s_inv
    W = gen_weights(layer.N, layer.K, seed, wl.config_id, key) if with_weights else None
    gi = act_order_gidx(layer.K, g, seed, wl.config_id, key) if wl.act_order else None
    return LayerInputs(layer.K, layer.N, M, wl.act_dtype, X, W, s, s_call, g, wl.symmetric, gi)


# ---- the decode step as a chain of projections ---------------------------------------
# One transformer block's projections in decode order, each fed from an earlier output.
# The non-GEMM parts of a block (attention, residual, normalisation, the gated MLP's
# activation) are not part of the W4A16 path; a fixed stand-in takes their place:
#   qkv      reads the block's input (the previous block's down output; the seeded X for
#            the first block);
#   o        reads the first 4096 values of the qkv output (the query slice stands in for
#            the attention output);
#   gate_up  reads the o output;
#   down     reads the first 11008 values of the gate_up output (the gate half stands in
#            for silu(gate) * up).
# CHAIN_SOURCE[j] = (index of the projection whose output is read, -1 for the block
# input, first column of the slice).
CHAIN_SOURCE = ((-1, 0), (0, 0), (1, 0), (2, 0))


def chain_gain(K: int) -> float:
    """A fixed per-layer gain standing in for the normalisation before each projection:
    with W ~ N(0, 0.02^2) a projection of K inputs multiplies the activations' size by
    about 0.02 sqrt(K), so its input is scaled by the inverse (folded into s_inv, as AWQ
    folds s^-1 into the preceding normalisation) and values stay O(1) through the chain."""
    return 1.0 / (W_STD * float(np.sqrt(K)))


def chain_s_inv(s_inv: np.ndarray) -> np.ndarray:
    """s_inv of a projection inside the decode chain: the layer's AWQ s^-1 times its gain."""
    K = s_inv.shape[0]
    return (s_inv.astype(np.float32) * np.float32(chain_gain(K))).astype(np.float32)


# ---- byte and flop accounting of the measurement -------------------------------------
def effective_weight_bytes(N: int, K: int, group_size: int, symmetric: bool,
                           has_gidx: bool) -> int:
    """Algorithmic bytes one GEMM must read for its weights: packed codes (0.5 B/weight),
    fp16 scales, fp16 zero points (asymmetric only) and the int32 g_idx vector."""
    G = K // group_size
    return N * K // 2 + 2 * G * N + (0 if symmetric else 2 * G * N) + (4 * K if has_gidx else 0)


def gemm_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


def roofline_tokens_per_s(bandwidth_gbs: float, model_gb: float) -> float:
    """Decode bound: every weight byte is read once per generated token."""
    return bandwidth_gbs / model_gb
