"""The C-ABI library builds, loads and exports what include/qsa.h declares;
host-side argument checks reject bad calls before any CUDA work (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qsa.h")


@pytest.fixture(scope="module")
def lib():
    from token_indexed_sparse_b200 import build, qsa
    build.build()
    return qsa.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(qsa_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("qsa_forward", "qsa_backward", "qsa_forward_workspace_size",
                     "qsa_backward_workspace_size", "qsa_status_string", "qsa_route_plan"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in enumerate(["QSA_OK", "QSA_ERR_INVALID_ARGUMENT", "QSA_ERR_UNSUPPORTED",
                                 "QSA_ERR_MISALIGNED", "QSA_ERR_WORKSPACE_TOO_SMALL", "QSA_ERR_CUDA"]):
        assert lib.qsa_status_string(code).decode() == name
    assert b"sm_100a" in lib.qsa_version()


def test_workspace_sizes(lib):
    fw = lib.qsa_forward_workspace_size(32768, 32768, 24, 2, 564)
    bw = lib.qsa_backward_workspace_size(32768, 32768, 24, 2, 564)
    assert fw >= 32768 * 564 * 4 and bw > fw
    assert fw % 256 == 0 and bw % 256 == 0
    # outside the supported envelope -> 0
    assert lib.qsa_forward_workspace_size(16, 16, 8, 1, 4) == 0        # 8 heads per KV head
    assert lib.qsa_forward_workspace_size(0, 16, 12, 1, 4) == 0
    assert lib.qsa_forward_workspace_size(16, 16, 12, 1, 16385) == 0
    assert lib.qsa_backward_workspace_size(2**30, 16, 12, 1, 4) == 0   # T * n_sel > INT32_MAX


def test_launch_counts(lib):
    # forward: route rows + attention; backward: route rows, five tile-list kernels,
    # dQ and one dK/dV launch that walks every query phase, whatever the sizes
    assert lib.qsa_launch_count(32768, 32768, 24, 2, 564, 0) == 2
    assert lib.qsa_launch_count(32768, 32768, 24, 2, 564, 1) == 7
    assert lib.qsa_launch_count(16384, 16384, 12, 1, 512, 1) == 7
    assert lib.qsa_launch_count(256, 256, 12, 1, 64, 1) == 7
    assert lib.qsa_launch_count(16, 16, 8, 1, 4, 1) == 0


def _fwd(lib, q=256, k=256, v=256, routes=256, T=16, T_kv=16, H=12, G=1, n_sel=4, scale=0.0625,
         out=256, lse=256, ws=256, ws_bytes=1 << 20):
    P = ctypes.c_void_p
    return lib.qsa_forward(P(q), P(k), P(v), P(routes), T, T_kv, H, G, n_sel, scale, P(out), P(lse),
                           P(ws), ws_bytes, None)


def test_host_validation_before_any_launch(lib):
    # These return before touching CUDA, so they run without a GPU.
    assert _fwd(lib, q=0) == 1                       # null pointer
    assert _fwd(lib, T=0) == 1
    assert _fwd(lib, n_sel=0) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, scale=float("inf")) == 1
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, scale=-1.0) == 1
    assert _fwd(lib, H=16, G=1) == 2                 # 16 query heads per KV head
    assert _fwd(lib, H=13, G=2) == 2
    assert _fwd(lib, q=264) == 3                     # 8-byte aligned BF16 tensor
    assert _fwd(lib, routes=258) == 3
    assert _fwd(lib, ws=4096 + 16) == 3
    assert _fwd(lib, ws_bytes=16) == 4
    P = ctypes.c_void_p
    st = lib.qsa_backward(P(256), P(256), P(256), P(256), P(256), P(256), P(256), 16, 16, 12, 1, 4,
                          0.0625, P(256), P(256), P(0), P(256), 1 << 30, None)
    assert st == 1                                   # null dv
    st = lib.qsa_backward(P(256), P(256), P(256), P(256), P(256), P(256), P(256), 16, 16, 12, 1, 4,
                          0.0625, P(256), P(256), P(256), P(256), 8, None)
    assert st == 4
    st = lib.qsa_route_plan(P(256), 16, 16, 4, P(256), P(256), P(256), P(260), P(256), 1 << 20, None)
    assert st == 3                                   # int64 entries need 8-byte alignment
    st = lib.qsa_tile_plan(P(256), 16, 16, 4, P(256), P(256), P(256), P(260), P(256), 1 << 20, None)
    assert st == 3
    st = lib.qsa_tile_plan(P(256), 16, 16, 4, P(256), P(0), P(256), P(256), P(256), 1 << 20, None)
    assert st == 1                                   # null row_cols
    st = lib.qsa_tile_plan(P(256), 16, 16, 4, P(256), P(256), P(256), P(256), P(256), 8, None)
    assert st == 4                                   # scratch too small
    assert lib.qsa_tile_plan_scratch_size(16, 300) == 2 * 256 + 256


def test_saved_and_kvwait_host_validation(lib):
    # the backward that reuses a forward's route lists checks the forward
    # workspace (present, 256-byte aligned, large enough) before any launch;
    # routes are not an argument there.  These return before touching CUDA.
    P = ctypes.c_void_p
    big = 1 << 30

    def saved(fws=4096, fws_bytes=big, ws=8192, ws_bytes=big, dv=256):
        return lib.qsa_backward_saved(P(256), P(256), P(256), P(256), P(256), P(256), P(fws), fws_bytes, 16, 16,
                                      12, 1, 4, 0.0625, P(256), P(256), P(dv), 0, P(ws), ws_bytes, None, None,
                                      None, 0)
    assert saved(fws=0) == 1
    assert saved(dv=0) == 1
    assert saved(fws=4096 + 16) == 3
    assert saved(fws_bytes=8) == 4
    assert saved(ws_bytes=8) == 4
    fwd_need = lib.qsa_forward_workspace_size(16, 16, 12, 1, 4)
    assert saved(fws_bytes=fwd_need - 1) == 4

    def kvwait_fwd(q=256, ws_bytes=big):
        return lib.qsa_forward_kvwait(P(q), P(256), P(256), P(256), 16, 16, 12, 1, 4, 0.0625, P(256), P(256),
                                      P(4096), ws_bytes, None, None, None, 0)
    assert kvwait_fwd(q=0) == 1 and kvwait_fwd(q=264) == 3 and kvwait_fwd(ws_bytes=8) == 4

    def kvwait_bwd(routes=256, kv_fp32=0, ws_bytes=big):
        return lib.qsa_backward_kvwait(P(256), P(256), P(256), P(256), P(256), P(256), P(routes), 16, 16, 12, 1,
                                       4, 0.0625, P(256), P(256), P(256), kv_fp32, P(4096), ws_bytes, None, None,
                                       None, 0)
    assert kvwait_bwd(routes=0) == 1 and kvwait_bwd(routes=258) == 3 and kvwait_bwd(kv_fp32=1, ws_bytes=8) == 4


def _fwd_noalloc(lib, q=256, T=16, n_sel=4):
    P = ctypes.c_void_p
    f = lib.qsa_forward_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_float, P, P, P]
    return f(P(q), P(256), P(256), P(256), T, T, 12, 1, n_sel, 0.0625, P(256), P(256), None)


def test_noalloc_host_validation_order(lib):
    # the allocation-free forward checks in qsa_forward's order: pointers, sizes,
    # scale, alignment, and only then its fixed scratch limit
    assert _fwd_noalloc(lib, q=0) == 1
    assert _fwd_noalloc(lib, T=0) == 1
    assert _fwd_noalloc(lib, q=264) == 3                          # misaligned, small
    assert _fwd_noalloc(lib, T=16384, n_sel=512) == 4             # aligned, needs ~32 MiB of scratch
    assert _fwd_noalloc(lib, q=264, T=16384, n_sel=512) == 3      # misaligned and too large


def test_bitmap_routes_host_validation(lib):
    P = ctypes.c_void_p

    def call(sel=256, lo=256, hi=256, bb=256, tb=256, T=8, NB=4, T_kv=16, bs=4, n_sel=16, routes=256,
             cnt=0, mx=0):
        return lib.qsa_bitmap_routes(P(sel), P(lo), P(hi), P(bb), P(tb), T, NB, T_kv, bs, n_sel, P(routes),
                                     P(cnt), P(mx), None)
    assert call(sel=0) == 1
    assert call(routes=0) == 1
    assert call(T=0) == 1 and call(NB=0) == 1 and call(T_kv=0) == 1 and call(n_sel=0) == 1
    assert call(bs=0) == 1
    assert call(T_kv=2**31) == 1
    assert call(T=2**30, n_sel=4) == 1                 # T * n_sel > INT32_MAX
    assert call(lo=258) == 3 and call(routes=258) == 3 and call(cnt=258) == 3
    assert call(sel=264) == 3                          # the bitmap is read with 16-byte loads


def test_selector_host_validation(lib):
    P = ctypes.c_void_p

    def scores(qi=256, kb=256, T=8, NB=4, Hi=64, Di=128, scale=0.5, sc=256, stride=4):
        return lib.qsa_selector_scores(P(qi), P(kb), T, NB, Hi, Di, scale, None, None, None, P(sc), stride, None,
                                       None)
    assert scores(qi=0) == 1 and scores(sc=0) == 1
    assert scores(T=0) == 1 and scores(stride=3) == 1 and scores(scale=0.0) == 1
    assert scores(Di=64) == 2 and scores(Hi=48) == 2 and scores(Hi=16) == 2
    assert scores(qi=264) == 3 and scores(sc=258) == 3

    def topk(sc=256, stride=4, T=8, NB=4, k=2, b=256, r=256):
        return lib.qsa_selector_topk(P(sc), stride, T, NB, k, None, None, None, P(b), P(r), None)
    assert topk(b=0) == 1 and topk(k=0) == 1 and topk(stride=2) == 1
    assert topk(r=258) == 3


def test_no_cpu_fallback_without_library(monkeypatch, tmp_path):
    from token_indexed_sparse_b200 import qsa
    monkeypatch.setattr(qsa, "_lib", None)
    monkeypatch.setattr(qsa, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        qsa.library()


def test_binding_refuses_output_buffers_the_kernels_would_overrun():
    # caller-provided outputs are written in place through their pointers: the
    # binding checks them before any call (CPU tensors stand in for the device)
    import torch
    from token_indexed_sparse_b200 import qsa
    dev = torch.device("cpu")
    ok = torch.empty(4, 12, 256, dtype=torch.bfloat16)
    assert qsa._out(ok, (4, 12, 256), torch.bfloat16, dev, "out") is ok
    with pytest.raises(ValueError, match="shape"):
        qsa._out(torch.empty(4, 12, 255, dtype=torch.bfloat16), (4, 12, 256), torch.bfloat16, dev, "out")
    with pytest.raises(TypeError):
        qsa._out(torch.empty(4, 12, 256, dtype=torch.float32), (4, 12, 256), torch.bfloat16, dev, "out")
    with pytest.raises(ValueError, match="contiguous"):
        qsa._out(torch.empty(12, 4, 256, dtype=torch.bfloat16).transpose(0, 1), (4, 12, 256), torch.bfloat16, dev,
                 "out")
    with pytest.raises(ValueError, match="on"):
        qsa._out(ok, (4, 12, 256), torch.bfloat16, torch.device("meta"), "out")
    ws = torch.empty(1024, dtype=torch.uint8)
    assert qsa._workspace(1024, dev, ws) is ws
    with pytest.raises(ValueError):
        qsa._workspace(1024, dev, torch.empty(256, dtype=torch.float32))
    with pytest.raises(ValueError):
        qsa._workspace(1024, dev, torch.empty(2048, dtype=torch.uint8)[::2])
