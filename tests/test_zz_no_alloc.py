"""qsa_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (an extension inside a host application that owns the device
allocator, or a latency-critical path that must not call cudaMalloc) get their
scratch from a fixed array inside the library instead of a caller workspace.
This file runs last so that a failure here leaves every other test already run.
The entry point is called through the C ABI twice in a row, on different
inputs (the second smaller than the first, so stale scratch from the first call
would show).  It runs the same kernels as qsa_forward on the same inputs, so
each result must equal qsa_forward's bit for bit; each is also checked against
the FP64 CPU oracle within the parity tolerances of the other GPU tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
REL_TOL = 1e-2
LSE_TOL = 1e-3
QSA_NOALLOC_SCRATCH_BYTES = 16 << 20


def _lib():
    lib = qsa.library()
    f = lib.qsa_forward_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_float, vp, vp, vp]
    return lib


def _call_noalloc(lib, q, k, v, routes, scale, out, lse):
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    T, H, _ = q.shape
    T_kv, G, _ = k.shape
    return lib.qsa_forward_noalloc(P(q), P(k), P(v), P(routes), T, T_kv, H, G, routes.shape[1], scale,
                                   P(out), P(lse), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _inputs(wl):
    routes = torch.from_numpy(np.array(W.make_routes(wl), dtype=np.int32)).to(DEV)
    q, k, v, _ = W.make_tensors(wl, with_grad=False)
    return q.to(DEV), k.to(DEV), v.to(DEV), routes


def _compare_oracle(out, lse, q, k, v, routes, scale):
    f = lambda x: x.float().cpu().numpy().astype(np.float64)  # noqa: E731
    ref_out, ref_lse = oracle.forward_dense(f(q), f(k), f(v), routes.cpu().numpy(), scale)
    err = np.abs(f(out) - ref_out).max() / max(np.abs(ref_out).max(), 1e-3)
    assert err <= REL_TOL
    got = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(got[~fin] == -np.inf)
    assert np.abs(got[fin] - ref_lse[fin]).max() <= LSE_TOL


def test_noalloc_forward_matches_workspace_forward_twice():
    lib = _lib()
    for wl in (W.WORKLOADS["seq4k"].scaled(1024), W.WORKLOADS["tiny"]):
        q, k, v, routes = _inputs(wl)
        assert qsa.forward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, wl.W) <= QSA_NOALLOC_SCRATCH_BYTES
        ref_out, ref_lse = qsa.forward(q, k, v, routes, wl.scale)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((wl.T, wl.H), float("nan"), device=DEV)
        assert _call_noalloc(lib, q, k, v, routes, wl.scale, out, lse) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(lse, ref_lse)
        _compare_oracle(out, lse, q, k, v, routes, wl.scale)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib()
    T, T_kv, n_sel = 16384, 16384, 512          # needs ~32 MiB of scratch
    assert qsa.forward_workspace_size(T, T_kv, 12, 1, n_sel) > QSA_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(T, 12, 256, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(T_kv, 1, 256, dtype=torch.bfloat16, device=DEV)
    routes = torch.full((T, n_sel), -1, dtype=torch.int32, device=DEV)
    out = torch.full_like(q, 3.0)
    lse = torch.full((T, 12), 3.0, device=DEV)
    assert _call_noalloc(lib, q, k, k, routes, 1.0 / 16, out, lse) == 4     # QSA_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert torch.all(out == 3.0) and torch.all(lse == 3.0)                  # nothing launched
