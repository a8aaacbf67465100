"""B200 (sm_100a) W4A16: 4-bit weight-only quantised linear layers with 16-bit activations.

Thin Python binding of the C ABI in include/w4a16.h.  The functions below carry the C
names, check each tensor's dtype and size, and marshal arguments: PyTorch provides
device memory, streams and output allocation; every step of the computation runs in
the library's CUDA kernels
(bit_weight_only_w4_b200/_lib/libw4a16.so, built in-tree by
``python -m bit_weight_only_w4_b200.build``).  There is no CPU fallback: if the library
is missing or a call fails, an exception is raised.

    qweight, scales, zeros = w4_quantize_pack(W, s, group_size=128)
    Y = w4a16_gemm(X, qweight, scales, zeros, group_size=128, s_inv=s_inv)
"""
import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libw4a16.so")

W4_OK, W4_ERR_INVALID_ARG, W4_ERR_UNSUPPORTED, W4_ERR_CUDA, W4_ERR_TIMEOUT, W4_ERR_DEVICE_ARG = range(6)
W4_F16, W4_BF16, W4_F32 = 0, 1, 2
W4_FP4_NVFP4, W4_FP4_MXFP4 = 0, 1
FP4_BLOCK = {W4_FP4_NVFP4: 16, W4_FP4_MXFP4: 32}

_lib = None
_lib_lock = threading.Lock()


class W4Error(RuntimeError):
    """A library call returned a status other than W4_OK."""

    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {w4_status_string(status)}")


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"W4A16 CUDA library not found at {LIB_PATH}; build it with "
                "`python -m bit_weight_only_w4_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, u64, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                 ctypes.c_uint64, ctypes.c_size_t)
        st = ctypes.c_int
        L.w4_quantize_pack.argtypes = [vp, st, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp]
        L.w4_quantize_pack.restype = st
        L.w4a16_gemm.argtypes = [vp, st, i64, i64, i64, vp, vp, vp, vp, i32, vp, vp, st, vp, sz, vp]
        L.w4a16_gemm.restype = st
        L.w4a16_gemm_noalloc.argtypes = [vp, st, i64, i64, i64, vp, vp, vp, vp, i32, vp, vp, st, vp]
        L.w4a16_gemm_noalloc.restype = st
        L.w4a16_workspace_bytes.argtypes = [i64, i64, i64, i32]
        L.w4a16_workspace_bytes.restype = sz
        L.w4_unpack_canonical.argtypes = [vp, i64, i64, vp, vp]
        L.w4_unpack_canonical.restype = st
        L.w4_check_device_error.argtypes = []
        L.w4_check_device_error.restype = st
        L.w4_set_wait_limit_ns.argtypes = [u64]
        L.w4_set_wait_limit_ns.restype = st
        L.w4_selftest_noalloc_scratch.argtypes = [i32, ctypes.POINTER(u64)]
        L.w4_selftest_noalloc_scratch.restype = st
        L.w4_selftest_expired_wait.argtypes = [vp]
        L.w4_selftest_expired_wait.restype = st
        L.w4_status_string.argtypes = [st]
        L.w4_status_string.restype = ctypes.c_char_p
        L.w4_actorder_perm.argtypes = [vp, i64, i32, vp, vp]
        L.w4_actorder_perm.restype = st
        L.w4_quantize_pack_perm.argtypes = [vp, st, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp]
        L.w4_quantize_pack_perm.restype = st
        L.w4a16_gemm_perm.argtypes = [vp, st, i64, i64, i64, vp, vp, vp, vp, i32, vp, vp, st, vp, sz, vp]
        L.w4a16_gemm_perm.restype = st
        L.w4a16_workspace_bytes_perm.argtypes = [i64, i64, i64, i32]
        L.w4a16_workspace_bytes_perm.restype = sz
        L.w4_awq_search.argtypes = [vp, st, i64, i64, vp, st, i64, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.w4_awq_search.restype = st
        L.w4_awq_search_workspace_bytes.argtypes = [i64, i64, i64, i32, i32, i32]
        L.w4_awq_search_workspace_bytes.restype = sz
        L.w4_fp4_quantize_pack.argtypes = [vp, st, i64, i64, st, vp, vp, vp, vp]
        L.w4_fp4_quantize_pack.restype = st
        L.w4a16_fp4_gemm.argtypes = [vp, st, i64, i64, i64, vp, vp, vp, st, vp, st, vp, sz, vp]
        L.w4a16_fp4_gemm.restype = st
        L.w4a16_fp4_workspace_bytes.argtypes = [i64, i64, i64, st]
        L.w4a16_fp4_workspace_bytes.restype = sz
        L.w4a16_gemm_chain.argtypes = [ctypes.POINTER(ChainLayer), i32, i64, st, st, vp, sz, vp]
        L.w4a16_gemm_chain.restype = st
        L.w4a16_chain_workspace_bytes.argtypes = [i64]
        L.w4a16_chain_workspace_bytes.restype = sz
        _lib = L
    return _lib


class ChainLayer(ctypes.Structure):
    """w4_chain_layer of include/w4a16.h."""
    _fields_ = [("X", ctypes.c_void_p), ("ldx", ctypes.c_int64), ("qweight", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p), ("s_inv", ctypes.c_void_p),
                ("Y", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("group_size", ctypes.c_int32)]


# ---------------------------------------------------------------- marshalling helpers
def _torch():
    import torch
    return torch


def _dtype_code(dt):
    torch = _torch()
    if dt == torch.float16:
        return W4_F16
    if dt == torch.bfloat16:
        return W4_BF16
    if dt == torch.float32:
        return W4_F32
    raise TypeError(f"unsupported dtype {dt}")


def _ptr(t):
    # c_void_p arguments take a plain int (or None for NULL)
    return None if t is None else t.data_ptr()


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, what):
    if status != W4_OK:
        raise W4Error(status, what)


def _need_cuda(*tensors):
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("tensors are on different devices")
    return dev


def _expect(t, name, dtypes, shape=None, numel=None):
    """Refuse a tensor of the wrong dtype or size before its pointer reaches the library,
    which sees only the pointer and would read past a short buffer."""
    if t is None:
        return
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, not {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must hold {numel} elements, not {t.numel()}")


def _matrix(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be a matrix, not of shape {tuple(t.shape)}")
    return t.shape


def _groups(K, group_size):
    if group_size <= 0 or K % group_size != 0:
        raise ValueError(f"group_size {group_size} must divide K = {K}")
    return K // group_size


def _f16s():
    torch = _torch()
    return (torch.float16, torch.bfloat16)


def _words():
    torch = _torch()
    return (torch.int32, torch.uint32)


class _DeviceGuard:
    def __init__(self, device):
        self.device = device

    def __enter__(self):
        torch = _torch()
        self.prev = torch.cuda.current_device()
        self.switch = self.prev != self.device.index
        if self.switch:
            torch.cuda.set_device(self.device)

    def __exit__(self, *exc):
        if self.switch:
            _torch().cuda.set_device(self.prev)


# ---------------------------------------------------------------- C ABI, same names
def w4_status_string(status):
    return lib().w4_status_string(int(status)).decode()


def w4a16_workspace_bytes(M, N, K, group_size):
    return int(lib().w4a16_workspace_bytes(int(M), int(N), int(K), int(group_size)))


def w4_actorder_perm(g_idx, group_size, perm=None, stream=None):
    """perm int32 [K]: the channels sorted by g_idx (ties in channel order), for packing
    act-order weights with contiguous groups (every group must hold group_size channels;
    otherwise w4_check_device_error() reports W4_ERR_DEVICE_ARG)."""
    torch = _torch()
    if g_idx.dim() != 1:
        raise ValueError("g_idx must be a vector")
    K = g_idx.shape[0]
    _expect(g_idx, "g_idx", (torch.int32,))
    _expect(perm, "perm", (torch.int32,), numel=K)
    dev = _need_cuda(g_idx, perm)
    if perm is None:
        perm = torch.empty(K, dtype=torch.int32, device=dev)
    with _DeviceGuard(dev):
        st = lib().w4_actorder_perm(_ptr(g_idx), K, int(group_size), _ptr(perm), _stream_handle(stream, dev))
    _check(st, "w4_actorder_perm")
    return perm


def w4_awq_search(W, X, group_size=128, symmetric=False, n_grid=20, stream=None):
    """AWQ's scale search on the calibration rows X [M,K] for W [N,K] (both CUDA, fp16 or
    bf16): candidates s = m^a / geomean(m^a), m the mean |X| per channel, a = j / n_grid.
    Returns (best j, its exponent a, host float64 losses [n_grid], s_best float32 [K] on
    the device).  Synchronous."""
    torch = _torch()
    N, K = _matrix(W, "W")
    M, KX = _matrix(X, "X")
    if KX != K:
        raise ValueError(f"X has {KX} channels, W has {K}")
    _expect(W, "W", _f16s())
    _expect(X, "X", _f16s())
    dev = _need_cuda(W, X)
    s_best = torch.empty(K, dtype=torch.float32, device=dev)
    losses = (ctypes.c_double * int(n_grid))()
    best = ctypes.c_int32(-1)
    with _DeviceGuard(dev):
        need = lib().w4_awq_search_workspace_bytes(M, N, K, int(group_size), int(bool(symmetric)), int(n_grid))
        if need == 0:
            raise ValueError("w4_awq_search: unsupported sizes")
        # a buffer of its own: the search writes over the front of its workspace, where the
        # cached GEMM workspace keeps the zero-filled split-K slots
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        st = lib().w4_awq_search(_ptr(W), _dtype_code(W.dtype), N, K, _ptr(X), _dtype_code(X.dtype), M,
                                 int(group_size), int(bool(symmetric)), int(n_grid), _ptr(s_best),
                                 ctypes.addressof(losses), ctypes.addressof(best), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream_handle(stream, dev))
    _check(st, "w4_awq_search")
    import numpy as np
    return best.value, best.value / n_grid, np.array(losses[:], dtype=np.float64), s_best


def w4_quantize_pack(W, s=None, group_size=128, symmetric=False, g_idx=None,
                     qweight=None, scales=None, zeros=None, stream=None, perm=None):
    """AWQ scaling + group-wise RTN INT4 + packing of W [N,K] (fp16/bf16, CUDA).

    With perm (from w4_actorder_perm; g_idx then None) column k of the packed matrix is
    channel perm[k] and groups are contiguous.  Returns (qweight uint32-as-int32 [N*K/8]
    device layout, scales fp16 [G,N], zeros fp16 [G,N] or None when symmetric)."""
    torch = _torch()
    N, K = _matrix(W, "W")
    G = _groups(K, group_size)
    if perm is not None and g_idx is not None:
        raise ValueError("pass g_idx or perm, not both")
    _expect(W, "W", _f16s())
    _expect(s, "s", (torch.float32,), numel=K)
    _expect(g_idx, "g_idx", (torch.int32,), numel=K)
    _expect(perm, "perm", (torch.int32,), numel=K)
    _expect(qweight, "qweight", _words(), numel=N * K // 8)
    _expect(scales, "scales", (torch.float16,), shape=(G, N))
    _expect(zeros, "zeros", (torch.float16,), shape=(G, N))
    dev = _need_cuda(W, s, g_idx, qweight, scales, zeros, perm)
    if qweight is None:
        qweight = torch.empty(N * K // 8, dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(G, N, dtype=torch.float16, device=dev)
    if zeros is None and not symmetric:
        zeros = torch.empty(G, N, dtype=torch.float16, device=dev)
    with _DeviceGuard(dev):
        if perm is not None:
            st = lib().w4_quantize_pack_perm(_ptr(W), _dtype_code(W.dtype), N, K, _ptr(s), int(group_size),
                                             int(bool(symmetric)), _ptr(perm), _ptr(qweight),
                                             _ptr(scales), _ptr(zeros), _stream_handle(stream, dev))
        else:
            st = lib().w4_quantize_pack(_ptr(W), _dtype_code(W.dtype), N, K, _ptr(s), int(group_size),
                                        int(bool(symmetric)), _ptr(g_idx), _ptr(qweight),
                                        _ptr(scales), _ptr(zeros), _stream_handle(stream, dev))
    _check(st, "w4_quantize_pack")
    return qweight, scales, zeros


_ws_cache = {}
_ws_lock = threading.Lock()


def workspace_for(device, nbytes):
    """A zero-initialised scratch buffer of at least nbytes on `device`, shared by every
    call on that device that passes no workspace of its own (the kernels leave it
    zero-filled where that matters).  Calls sharing it must be ordered on the GPU."""
    torch = _torch()
    key = torch.device(device).index
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            _ws_cache[key] = buf
        return buf


_DTYPES = None


def _dtypes():
    """(float16, bfloat16, float32, int32, uint32), looked up once."""
    global _DTYPES
    if _DTYPES is None:
        torch = _torch()
        _DTYPES = (torch.float16, torch.bfloat16, torch.float32, torch.int32, torch.uint32)
    return _DTYPES


def _gemm_args(X, qweight, scales, zeros, group_size, g_idx, s_inv, Y, perm=None):
    """Shapes and dtypes of a GEMM call; returns (M, K, N), N taken from the scales.  A
    well-formed call passes one combined test (the decode path is called per token and
    per layer); any failure goes through the per-tensor checks, which name the culprit."""
    f16, bf16, f32, i32, u32 = _dtypes()
    xs, ss = X.shape, scales.shape
    if len(xs) == 2 and len(ss) == 2 and group_size > 0 and xs[1] % group_size == 0:
        M, K = xs
        N = ss[1]
        if ((X.dtype is f16 or X.dtype is bf16)
                and (qweight.dtype is i32 or qweight.dtype is u32) and qweight.numel() == N * K // 8
                and scales.dtype is f16 and ss[0] == K // group_size
                and (zeros is None or (zeros.dtype is f16 and zeros.shape == ss))
                and (g_idx is None or (g_idx.dtype is i32 and g_idx.numel() == K))
                and (s_inv is None or (s_inv.dtype is f32 and s_inv.numel() == K))
                and (perm is None or (perm.dtype is i32 and perm.numel() == K))
                and (Y is None or ((Y.dtype is f16 or Y.dtype is bf16 or Y.dtype is f32)
                                   and Y.shape == (M, N)))):
            return M, K, N
    _gemm_args_checked(X, qweight, scales, zeros, group_size, g_idx, s_inv, Y, perm)
    raise ValueError("inconsistent GEMM arguments")


def _gemm_args_checked(X, qweight, scales, zeros, group_size, g_idx, s_inv, Y, perm=None):
    torch = _torch()
    M, K = _matrix(X, "X")
    G = _groups(K, group_size)
    N = _matrix(scales, "scales")[1]
    _expect(X, "X", _f16s())
    _expect(qweight, "qweight", _words(), numel=N * K // 8)
    _expect(scales, "scales", (torch.float16,), shape=(G, N))
    _expect(zeros, "zeros", (torch.float16,), shape=(G, N))
    _expect(g_idx, "g_idx", (torch.int32,), numel=K)
    _expect(s_inv, "s_inv", (torch.float32,), numel=K)
    _expect(Y, "Y", _f16s() + (torch.float32,), shape=(M, N))
    _expect(perm, "perm", (torch.int32,), numel=K)


def w4a16_gemm(X, qweight, scales, zeros, group_size=128, g_idx=None, s_inv=None,
               out_dtype=None, Y=None, workspace=None, stream=None, perm=None):
    """Y[M,N] = (X * s_inv)[M,K] @ dequant(qweight, scales, zeros, g_idx)^T on the GPU.

    With perm, the weights were packed with that permutation (w4_quantize_pack(perm=...))
    and the activation columns are gathered through it (w4a16_gemm_perm).

    Without `workspace`, every call on a device shares one cached zero-filled buffer, which
    is safe for calls ordered on one stream.  Calls that may run concurrently (unordered
    streams) must each pass a workspace of their own: torch.zeros(w4a16_workspace_bytes(...),
    dtype=torch.uint8, device=...)."""
    torch = _torch()
    M, K, N = _gemm_args(X, qweight, scales, zeros, group_size, g_idx, s_inv, Y, perm)
    if perm is not None and g_idx is not None:
        raise ValueError("pass g_idx or perm, not both")
    dev = _need_cuda(X, qweight, scales, zeros, g_idx, s_inv, Y, workspace, perm)
    out_dtype = out_dtype or X.dtype
    if Y is None:
        Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    with _DeviceGuard(dev):
        if perm is not None:
            need = lib().w4a16_workspace_bytes_perm(M, N, K, int(group_size)) if M > 0 else 0
        else:
            need = w4a16_workspace_bytes(M, N, K, group_size) if M > 0 else 0
        if workspace is None and need > 0:
            workspace = workspace_for(dev, need)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        if perm is not None:
            st = lib().w4a16_gemm_perm(_ptr(X), _dtype_code(X.dtype), M, N, K, _ptr(qweight), _ptr(scales),
                                       _ptr(zeros), _ptr(perm), int(group_size), _ptr(s_inv), _ptr(Y),
                                       _dtype_code(Y.dtype), _ptr(workspace), ws_bytes,
                                       _stream_handle(stream, dev))
        else:
            st = lib().w4a16_gemm(_ptr(X), _dtype_code(X.dtype), M, N, K, _ptr(qweight), _ptr(scales),
                                  _ptr(zeros), _ptr(g_idx), int(group_size), _ptr(s_inv), _ptr(Y),
                                  _dtype_code(Y.dtype), _ptr(workspace), ws_bytes,
                                  _stream_handle(stream, dev))
    _check(st, "w4a16_gemm_perm" if perm is not None else "w4a16_gemm")
    return Y


def w4a16_gemm_noalloc(X, qweight, scales, zeros, group_size=128, g_idx=None, s_inv=None,
                       out_dtype=None, Y=None, stream=None):
    """w4a16_gemm without a workspace, for callers that cannot allocate device memory at
    the point of the call: the library's fixed per-device scratch is used instead.  Only
    Y is allocated here, and only when not passed in."""
    torch = _torch()
    M, K, N = _gemm_args(X, qweight, scales, zeros, group_size, g_idx, s_inv, Y)
    dev = _need_cuda(X, qweight, scales, zeros, g_idx, s_inv, Y)
    out_dtype = out_dtype or X.dtype
    if Y is None:
        Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    with _DeviceGuard(dev):
        st = lib().w4a16_gemm_noalloc(_ptr(X), _dtype_code(X.dtype), M, N, K, _ptr(qweight),
                                      _ptr(scales), _ptr(zeros), _ptr(g_idx), int(group_size),
                                      _ptr(s_inv), _ptr(Y), _dtype_code(Y.dtype),
                                      _stream_handle(stream, dev))
    _check(st, "w4a16_gemm_noalloc")
    return Y


def _fp4_format(fmt):
    if fmt in ("nvfp4", W4_FP4_NVFP4):
        return W4_FP4_NVFP4
    if fmt in ("mxfp4", W4_FP4_MXFP4):
        return W4_FP4_MXFP4
    raise ValueError(f"unknown FP4 format {fmt!r} (nvfp4 or mxfp4)")


def w4_fp4_quantize_pack(W, fmt="nvfp4", qweight=None, block_scales=None, tensor_scale=None,
                         stream=None):
    """Quantise W [N,K] (fp16/bf16) to NVFP4 or MXFP4.  Returns (qweight int32 [N*K/8]
    in the device layout, block_scales uint8 [K/B, N], tensor_scale fp32 [1] or None)."""
    torch = _torch()
    f = _fp4_format(fmt)
    B = FP4_BLOCK[f]
    _matrix(W, "W")
    _expect(W, "W", _f16s())
    N, K = W.shape
    if K % B != 0:
        raise ValueError(f"K = {K} must be a multiple of the block ({B})")
    _expect(qweight, "qweight", _words(), numel=N * K // 8)
    _expect(block_scales, "block_scales", (torch.uint8,), shape=(K // B, N))
    _expect(tensor_scale, "tensor_scale", (torch.float32,), numel=1)
    dev = _need_cuda(W, qweight, block_scales, tensor_scale)
    if qweight is None:
        qweight = torch.empty(N * K // 8, dtype=torch.int32, device=dev)
    if block_scales is None:
        block_scales = torch.empty(K // B, N, dtype=torch.uint8, device=dev)
    if f == W4_FP4_NVFP4 and tensor_scale is None:
        tensor_scale = torch.empty(1, dtype=torch.float32, device=dev)
    if f == W4_FP4_MXFP4:
        tensor_scale = None
    with _DeviceGuard(dev):
        st = lib().w4_fp4_quantize_pack(_ptr(W), _dtype_code(W.dtype), N, K, f, _ptr(qweight),
                                        _ptr(block_scales), _ptr(tensor_scale), _stream_handle(stream, dev))
    _check(st, "w4_fp4_quantize_pack")
    return qweight, block_scales, tensor_scale


def w4a16_fp4_workspace_bytes(M, N, K, fmt="nvfp4"):
    return int(lib().w4a16_fp4_workspace_bytes(int(M), int(N), int(K), _fp4_format(fmt)))


def w4a16_fp4_gemm(X, qweight, block_scales, tensor_scale=None, fmt="nvfp4", out_dtype=None, Y=None,
                   workspace=None, stream=None):
    """Y = X @ What^T with NVFP4 / MXFP4 weights from w4_fp4_quantize_pack (fp16 X)."""
    torch = _torch()
    f = _fp4_format(fmt)
    B = FP4_BLOCK[f]
    _matrix(X, "X")
    _expect(X, "X", _f16s())
    M, K = X.shape
    if K % B != 0:
        raise ValueError(f"K = {K} must be a multiple of the block ({B})")
    N = block_scales.shape[1]
    _expect(qweight, "qweight", _words(), numel=N * K // 8)
    _expect(block_scales, "block_scales", (torch.uint8,), shape=(K // B, N))
    _expect(tensor_scale, "tensor_scale", (torch.float32,), numel=1)
    _expect(Y, "Y", (torch.float16, torch.bfloat16, torch.float32), shape=(M, N))
    dev = _need_cuda(X, qweight, block_scales, tensor_scale, Y, workspace)
    out_dtype = out_dtype or (Y.dtype if Y is not None else X.dtype)
    if Y is None:
        Y = torch.empty(M, N, dtype=out_dtype, device=dev)
    with _DeviceGuard(dev):
        need = w4a16_fp4_workspace_bytes(M, N, K, f) if M > 0 else 0
        if workspace is None and need > 0:
            workspace = workspace_for(dev, need)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().w4a16_fp4_gemm(_ptr(X), _dtype_code(X.dtype), M, N, K, _ptr(qweight), _ptr(block_scales),
                                  _ptr(tensor_scale), f, _ptr(Y), _dtype_code(Y.dtype), _ptr(workspace),
                                  ws_bytes, _stream_handle(stream, dev))
    _check(st, "w4a16_fp4_gemm")
    return Y


def w4a16_chain_workspace_bytes(M):
    return int(lib().w4a16_chain_workspace_bytes(int(M)))


def w4a16_gemm_chain(layers, workspace=None, stream=None):
    """Run a list of small-batch GEMMs (M <= 8) in order, in one persistent launch per 32
    layers.  Each layer is a dict with X, qweight, scales, zeros, group_size, s_inv and Y
    (X [M,K] may be a view of an earlier layer's Y: rows may be further apart than K,
    elements must be contiguous).  Layer l+1 reads its X only after every earlier output
    is stored.  Outputs are written into the given Y tensors; returns the list of Ys."""
    torch = _torch()
    n = len(layers)
    if n == 0:
        return []
    arr = (ChainLayer * n)()
    M = None
    act = None
    out = None
    devs = []
    for i, d in enumerate(layers):
        X, Y = d["X"], d["Y"]
        qw, sc, zr, s_inv = d["qweight"], d["scales"], d.get("zeros"), d.get("s_inv")
        g = int(d.get("group_size", 128))
        if X.dim() != 2 or Y.dim() != 2 or X.stride(1) != 1 or not Y.is_contiguous():
            raise ValueError(f"layer {i}: X must be a 2-D row-strided view, Y a contiguous matrix")
        m, K = X.shape
        N = Y.shape[1]
        if M is None:
            M, act, out = m, X.dtype, Y.dtype
        if m != M or Y.shape[0] != M or X.dtype != act or Y.dtype != out:
            raise ValueError(f"layer {i}: every layer has the same M, activation and output dtype")
        _expect(qw, "qweight", _words(), numel=N * K // 8)
        G = _groups(K, g)
        _expect(sc, "scales", _f16s(), shape=(G, N))
        _expect(zr, "zeros", _f16s(), shape=(G, N))
        _expect(s_inv, "s_inv", (torch.float32,), numel=K)
        if not X.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
        devs += [Y, qw, sc, zr, s_inv]
        arr[i] = ChainLayer(_ptr(X), X.stride(0), _ptr(qw), _ptr(sc), _ptr(zr), _ptr(s_inv), _ptr(Y),
                            N, K, g)
    dev = _need_cuda(*devs, workspace)
    if any(d["X"].device != dev for d in layers):
        raise ValueError("tensors are on different devices")
    with _DeviceGuard(dev):
        need = w4a16_chain_workspace_bytes(M)
        if workspace is None and need > 0:
            workspace = workspace_for(dev, need)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().w4a16_gemm_chain(arr, n, M, _dtype_code(act), _dtype_code(out), _ptr(workspace),
                                    ws_bytes, _stream_handle(stream, dev))
    _check(st, "w4a16_gemm_chain")
    return [d["Y"] for d in layers]


def w4_unpack_canonical(qweight, N, K, out=None, stream=None):
    torch = _torch()
    _expect(qweight, "qweight", _words(), numel=N * K // 8)
    _expect(out, "out", _words(), numel=N * K // 8)
    dev = _need_cuda(qweight, out)
    if out is None:
        out = torch.empty(N, K // 8, dtype=torch.int32, device=dev)
    with _DeviceGuard(dev):
        st = lib().w4_unpack_canonical(_ptr(qweight), int(N), int(K), _ptr(out),
                                       _stream_handle(stream, dev))
    _check(st, "w4_unpack_canonical")
    return out


def w4_check_device_error():
    """Synchronise the current device and raise if a kernel reported an error.  After a
    timeout the library zeroes its allocation-free scratch again, and this binding zeroes
    its cached workspace of the current device (a kernel that gave up a wait may have left
    split-K flags in either)."""
    st = lib().w4_check_device_error()
    if st == W4_ERR_TIMEOUT:
        torch = _torch()
        with _ws_lock:
            buf = _ws_cache.get(torch.cuda.current_device())
            if buf is not None:
                buf.zero_()
                torch.cuda.synchronize()
    _check(st, "w4_check_device_error")


def w4_set_wait_limit_ns(ns):
    _check(lib().w4_set_wait_limit_ns(int(ns)), "w4_set_wait_limit_ns")


def w4_selftest_expired_wait(stream=None):
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().w4_selftest_expired_wait(_stream_handle(stream, dev)), "w4_selftest_expired_wait")
