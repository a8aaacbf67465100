"""Host-side checks of the C ABI: the sm_100a library builds, loads, exports every entry
point declared in include/w4a16.h, and rejects bad arguments before touching a GPU.
No compute call is made (this file runs without a GPU)."""
import ctypes
import os
import re

import pytest

import bit_weight_only_w4_b200 as w4
from bit_weight_only_w4_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return w4.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "w4a16.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(w4\w*)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("w4_quantize_pack", "w4a16_gemm", "w4a16_workspace_bytes", "w4_unpack_canonical",
              "w4_check_device_error", "w4_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    # and nothing is hidden behind C++ mangling
    out = os.popen(f"nm -D --defined-only {w4.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, re.M), name


def test_status_strings(L):
    assert w4.w4_status_string(0) == "W4_OK"
    assert w4.w4_status_string(2) == "W4_ERR_UNSUPPORTED"
    assert w4.w4_status_string(99) == "W4_ERR_UNKNOWN"


def _gemm(L, M=1, N=128, K=128, g=128, X=16, qw=16, sc=16, Y=16, act=0, out=0, gidx=None):
    v = ctypes.c_void_p
    return L.w4a16_gemm(v(X), act, M, N, K, v(qw), v(sc), None, v(gidx) if gidx else None, g,
                        None, v(Y), out, v(256), 1 << 30, None)


def test_gemm_rejects_bad_shapes_before_launch(L):
    assert _gemm(L, N=8) == w4.W4_ERR_UNSUPPORTED            # N % 16
    assert _gemm(L, K=96, g=32) == w4.W4_ERR_UNSUPPORTED     # K % 64
    assert _gemm(L, K=128, g=48) == w4.W4_ERR_INVALID_ARG    # K % g
    assert _gemm(L, K=192, g=96) == w4.W4_ERR_UNSUPPORTED    # g not 32 or 64j
    assert _gemm(L, N=0) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, M=-1) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, act=2) == w4.W4_ERR_INVALID_ARG          # fp32 activations
    assert _gemm(L, out=7) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, M=0) == w4.W4_OK                         # empty batch: no-op


def test_gemm_rejects_null_and_misaligned_pointers(L):
    assert _gemm(L, X=0) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, Y=0) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, X=24) == w4.W4_ERR_INVALID_ARG           # not 16-byte aligned
    assert _gemm(L, qw=20) == w4.W4_ERR_INVALID_ARG
    assert _gemm(L, act=1, gidx=16) == w4.W4_ERR_UNSUPPORTED  # bf16 + act-order


def test_quantize_rejects_bad_arguments(L):
    v = ctypes.c_void_p
    q = L.w4_quantize_pack
    # symmetric with zeros / asymmetric without zeros
    assert q(v(16), 0, 16, 64, None, 32, 1, None, v(16), v(16), v(16), None) == w4.W4_ERR_INVALID_ARG
    assert q(v(16), 0, 16, 64, None, 32, 0, None, v(16), v(16), None, None) == w4.W4_ERR_INVALID_ARG
    assert q(None, 0, 16, 64, None, 32, 0, None, v(16), v(16), v(16), None) == w4.W4_ERR_INVALID_ARG
    assert q(v(16), 2, 16, 64, None, 32, 0, None, v(16), v(16), v(16), None) == w4.W4_ERR_INVALID_ARG
    assert q(v(16), 0, 15, 64, None, 32, 0, None, v(16), v(16), v(16), None) == w4.W4_ERR_UNSUPPORTED
    # too many groups for the shared-memory tables
    assert q(v(16), 0, 16, 64 * 1600, None, 32, 0, None, v(16), v(16), v(16), None) == \
        w4.W4_ERR_UNSUPPORTED


def test_workspace_bytes_invalid_sizes(L):
    assert w4.w4a16_workspace_bytes(1, 8, 128, 128) == 0
    assert w4.w4a16_workspace_bytes(0, 128, 128, 128) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    W = torch.zeros(16, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        w4.w4_quantize_pack(W, group_size=32)


def test_actorder_entry_points_reject_bad_arguments(L):
    v = ctypes.c_void_p
    # w4_actorder_perm: pointers, K % group_size
    assert L.w4_actorder_perm(None, 128, 32, v(256), None) == w4.W4_ERR_INVALID_ARG
    assert L.w4_actorder_perm(v(256), 128, 32, None, None) == w4.W4_ERR_INVALID_ARG
    assert L.w4_actorder_perm(v(256), 100, 32, v(256), None) == w4.W4_ERR_INVALID_ARG
    assert L.w4_actorder_perm(v(256), 128, 0, v(256), None) == w4.W4_ERR_INVALID_ARG
    # w4_quantize_pack_perm: perm is required
    assert L.w4_quantize_pack_perm(v(16), 0, 16, 64, None, 32, 1, None, v(16), v(16), None, None) == \
        w4.W4_ERR_INVALID_ARG
    # w4a16_gemm_perm: perm and workspace are required, shapes as w4a16_gemm
    g = L.w4a16_gemm_perm
    assert g(v(16), 0, 1, 128, 128, v(16), v(16), None, None, 128, None, v(16), 0, v(256), 1 << 30,
             None) == w4.W4_ERR_INVALID_ARG
    assert g(v(16), 0, 1, 128, 128, v(16), v(16), None, v(16), 128, None, v(16), 0, None, 1 << 30,
             None) == w4.W4_ERR_INVALID_ARG
    assert g(v(16), 0, 1, 8, 128, v(16), v(16), None, v(16), 128, None, v(16), 0, v(256), 1 << 30,
             None) == w4.W4_ERR_UNSUPPORTED
    assert g(v(16), 0, 0, 128, 128, None, None, None, None, 128, None, None, 0, None, 0, None) == w4.W4_OK
    assert L.w4a16_workspace_bytes_perm(1, 8, 128, 128) == 0
    assert L.w4a16_workspace_bytes_perm(0, 128, 128, 128) == 0


def test_awq_search_rejects_bad_arguments(L):
    """Every case below is refused by the host checks, before any CUDA call."""
    v = ctypes.c_void_p
    ok = dict(W=v(256), wd=0, N=128, K=256, X=v(256), xd=0, M=8, g=128, sym=0, n_grid=4, s=v(256),
              losses=v(256), best=v(256), ws=v(256), wsb=1 << 30)

    def call(**kw):
        a = dict(ok, **kw)
        return L.w4_awq_search(a["W"], a["wd"], a["N"], a["K"], a["X"], a["xd"], a["M"], a["g"], a["sym"],
                               a["n_grid"], a["s"], a["losses"], a["best"], a["ws"], a["wsb"], None)

    for bad in ("W", "X", "s", "losses", "best", "ws"):
        assert call(**{bad: None}) == w4.W4_ERR_INVALID_ARG, bad
    assert call(wd=2) == w4.W4_ERR_INVALID_ARG           # fp32 weights
    assert call(xd=7) == w4.W4_ERR_INVALID_ARG
    assert call(sym=2) == w4.W4_ERR_INVALID_ARG
    for M in (0, -1, (1 << 19) + 1):
        assert call(M=M) == w4.W4_ERR_INVALID_ARG, M
    for n_grid in (0, 1025):
        assert call(n_grid=n_grid) == w4.W4_ERR_INVALID_ARG, n_grid
    assert call(K=200) == w4.W4_ERR_INVALID_ARG          # K % group_size
    assert call(N=8) == w4.W4_ERR_UNSUPPORTED            # N % 16
    assert call(W=v(258)) == w4.W4_ERR_INVALID_ARG       # 16-byte alignment
    assert call(X=v(264)) == w4.W4_ERR_INVALID_ARG
    assert call(s=v(258)) == w4.W4_ERR_INVALID_ARG
    assert call(ws=v(272)) == w4.W4_ERR_INVALID_ARG      # 256-byte alignment
    ws = L.w4_awq_search_workspace_bytes
    assert ws(0, 128, 256, 128, 0, 4) == 0
    assert ws(8, 128, 256, 128, 0, 0) == 0
    assert ws(8, 128, 256, 128, 0, 1025) == 0
    assert ws(8, 8, 256, 128, 0, 4) == 0


def test_binding_refuses_wrong_dtypes_and_sizes():
    """The binding checks every tensor's dtype and size before its pointer reaches the
    library (which could not tell a short buffer from a long one).  CPU tensors suffice:
    the checks run before the device check."""
    import torch
    M, N, K, g = 2, 32, 256, 64
    G = K // g
    X = torch.zeros(M, K, dtype=torch.float16)
    qw = torch.zeros(N * K // 8, dtype=torch.int32)
    sc = torch.zeros(G, N, dtype=torch.float16)
    si = torch.zeros(K, dtype=torch.float32)
    gi = torch.zeros(K, dtype=torch.int32)

    def gemm(**kw):
        a = dict(X=X, qweight=qw, scales=sc, zeros=sc, group_size=g)
        a.update(kw)
        return w4.w4a16_gemm(**a)

    bad = [
        (TypeError, "qweight", dict(qweight=qw.to(torch.int64))),
        (ValueError, "qweight", dict(qweight=qw[:-1])),
        (ValueError, "scales", dict(scales=sc[:-1], zeros=None)),
        (ValueError, "zeros", dict(zeros=sc[:, :-1])),
        (TypeError, "scales", dict(scales=sc.to(torch.bfloat16), zeros=None)),
        (TypeError, "s_inv", dict(s_inv=si.half())),
        (ValueError, "s_inv", dict(s_inv=si[:-1])),
        (TypeError, "g_idx", dict(g_idx=gi.long())),
        (ValueError, "g_idx", dict(g_idx=gi[:-1])),
        (ValueError, "perm", dict(perm=gi[:-1])),
        (ValueError, "Y", dict(Y=torch.zeros(M, N + 1, dtype=torch.float16))),
        (TypeError, "Y", dict(Y=torch.zeros(M, N, dtype=torch.float64))),
        (TypeError, "X", dict(X=X.float())),
        (ValueError, "X", dict(X=X.reshape(-1))),
        (ValueError, "group_size", dict(group_size=96)),
        (ValueError, "group_size", dict(group_size=0)),
    ]
    for exc, what, kw in bad:
        with pytest.raises(exc, match=what):
            gemm(**kw)
        if "perm" not in kw:
            a = dict(X=X, qweight=qw, scales=sc, zeros=sc, group_size=g)
            a.update(kw)
            with pytest.raises(exc, match=what):
                w4.w4a16_gemm_noalloc(**a)
    with pytest.raises(ValueError, match="CUDA"):    # well-formed: stops at the device check
        gemm(s_inv=si, Y=torch.zeros(M, N, dtype=torch.float16))

    W = torch.zeros(N, K, dtype=torch.float16)
    for exc, what, kw in [
        (ValueError, "W", dict(W=W.reshape(-1))),
        (TypeError, "W", dict(W=W.float())),
        (ValueError, "s", dict(s=si[:-1])),
        (ValueError, "perm", dict(perm=gi[:-1])),
        (ValueError, "qweight", dict(qweight=qw[:-1])),
        (ValueError, "scales", dict(scales=sc[:, :-1])),
        (ValueError, "group_size", dict(group_size=100)),
    ]:
        a = dict(W=W, group_size=g)
        a.update(kw)
        with pytest.raises(exc, match=what):
            w4.w4_quantize_pack(**a)

    with pytest.raises(ValueError, match="channels"):
        w4.w4_awq_search(W, torch.zeros(M, K + 64, dtype=torch.float16), g)
    with pytest.raises(TypeError, match="X"):
        w4.w4_awq_search(W, torch.zeros(M, K, dtype=torch.float32), g)
    with pytest.raises(ValueError, match="vector"):
        w4.w4_actorder_perm(gi.reshape(2, -1), g)
    with pytest.raises(ValueError, match="perm"):
        w4.w4_actorder_perm(gi, g, perm=gi[:-1])
    with pytest.raises(ValueError, match="out"):
        w4.w4_unpack_canonical(qw, N, K, out=qw[:-1])


def test_chain_rejects_bad_arguments(L):
    """w4a16_gemm_chain checks its layer list before any CUDA call."""
    Lc = w4.ChainLayer

    def layer(**kw):
        d = dict(X=256, ldx=256, qweight=256, scales=256, zeros=256, s_inv=None, Y=256, N=256,
                 K=256, group_size=128)
        d.update(kw)
        return Lc(**d)

    def call(layers, M=1, act=0, out=0):
        arr = (Lc * len(layers))(*layers)
        return L.w4a16_gemm_chain(arr, len(layers), M, act, out, ctypes.c_void_p(256), 1 << 30, None)

    assert L.w4a16_gemm_chain(None, 1, 1, 0, 0, None, 0, None) == w4.W4_ERR_INVALID_ARG
    assert call([layer()], M=9) == w4.W4_ERR_UNSUPPORTED          # one token tile only
    assert call([layer()], act=2) == w4.W4_ERR_INVALID_ARG        # fp32 activations
    assert call([layer(ldx=128)]) == w4.W4_ERR_INVALID_ARG        # rows shorter than K
    assert call([layer(ldx=260)]) == w4.W4_ERR_INVALID_ARG        # rows not 16-byte apart
    assert call([layer(X=0)]) == w4.W4_ERR_INVALID_ARG            # NULL activations
    assert call([layer(X=258)]) == w4.W4_ERR_INVALID_ARG          # misaligned
    assert call([layer(N=8)]) == w4.W4_ERR_UNSUPPORTED            # N % 16
    assert call([layer(), layer(group_size=32)]) == w4.W4_ERR_UNSUPPORTED   # two group modes
    assert call([layer(K=65536, ldx=65536)], M=8) == w4.W4_ERR_UNSUPPORTED  # X' not resident
    assert call([], M=1) == w4.W4_OK                                 # nothing to do
    assert L.w4a16_chain_workspace_bytes(0) == 0 and L.w4a16_chain_workspace_bytes(9) == 0


def test_fp4_entry_points_reject_bad_arguments(L):
    """The FP4 quantiser and GEMM check formats, shapes and pointers before any CUDA call."""
    v = ctypes.c_void_p
    q = lambda **kw: L.w4_fp4_quantize_pack(  # noqa: E731
        v(kw.get("W", 256)), kw.get("wdt", 0), kw.get("N", 256), kw.get("K", 256), kw.get("fmt", 0),
        v(kw.get("qw", 256)), v(kw.get("bs", 256)),
        None if kw.get("ts", 256) is None else v(kw.get("ts", 256)), None)
    assert q(fmt=2) == w4.W4_ERR_INVALID_ARG                  # no such format
    assert q(fmt=1) == w4.W4_ERR_INVALID_ARG                  # MXFP4 has no tensor scale
    assert q(fmt=0, ts=None) == w4.W4_ERR_INVALID_ARG         # NVFP4 needs one
    assert q(wdt=2) == w4.W4_ERR_INVALID_ARG                  # fp32 weights
    assert q(N=8) == w4.W4_ERR_UNSUPPORTED                    # N % 16
    assert q(K=96) == w4.W4_ERR_UNSUPPORTED                   # K % 64
    assert q(W=0) == w4.W4_ERR_INVALID_ARG
    g = lambda **kw: L.w4a16_fp4_gemm(  # noqa: E731
        v(kw.get("X", 256)), kw.get("act", 0), kw.get("M", 1), kw.get("N", 256), kw.get("K", 256),
        v(256), v(kw.get("bs", 256)), None if kw.get("ts", 256) is None else v(kw.get("ts", 256)),
        kw.get("fmt", 0), v(256), kw.get("out", 0), v(256), 1 << 30, None)
    assert g(act=1) == w4.W4_ERR_UNSUPPORTED                  # bf16 activations
    assert g(act=2) == w4.W4_ERR_INVALID_ARG
    assert g(fmt=1) == w4.W4_ERR_INVALID_ARG                  # MXFP4 with a tensor scale
    assert g(ts=None) == w4.W4_ERR_INVALID_ARG                # NVFP4 without
    assert g(X=264) == w4.W4_ERR_INVALID_ARG                  # misaligned
    assert g(M=0) == w4.W4_OK
    assert L.w4a16_fp4_workspace_bytes(1, 8, 256, 0) == 0


def test_library_builds_without_warnings(L):
    """nvcc's log of the in-tree build holds no warning (an unused function, a narrowing
    conversion, a missing return...).  ptxas reports no spill in the decode kernels with
    one, four or eight token tiles, the fp16 layer-sequence kernel with 128-multiple
    groups (the decode step's), the prefill kernels and the quantisers, and at most 24
    bytes a thread in the two-tile decode kernels and the other layer-sequence kernels,
    which run at a 96-register cap."""
    log = open(os.path.join(os.path.dirname(w4.LIB_PATH), "build.log")).read()
    assert "warning" not in log.lower()
    name, seen = None, {}
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            name = m.group(1)
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            seen[name] = (int(m.group(1)), int(m.group(2)))
    assert seen
    for fn, (st, ld) in seen.items():
        strict = any(k in fn for k in ("decode_kernelILi1E", "decode_kernelILi4E", "decode_kernelILi8E",
                                        "prefill_kernel", "quantize", "fp4_pack", "chain_kernelILb0ELi0E",
                                        "prep_acts"))
        limit = 0 if strict else 24
        assert st <= limit and ld <= limit, (fn, st, ld)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library the package raises; it never falls back to a CPU path."""
    monkeypatch.setattr(w4, "LIB_PATH", str(tmp_path / "libw4a16.so"))
    monkeypatch.setattr(w4, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        w4.lib()
    with pytest.raises(RuntimeError, match="not found"):
        w4.w4a16_workspace_bytes(1, 128, 128, 128)
