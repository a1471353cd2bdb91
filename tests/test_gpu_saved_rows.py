"""qsa_backward_saved: the backward that reuses the forward's route lists.

It must return bit for bit what the backward that sorts the routes itself
returns, whether the forward's workspace is a separate buffer or the
backward's own, for BF16 and FP32 dK/dV, on rows with duplicates, invalid IDs
and empty rows.
"""
import numpy as np
import pytest
import torch

from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(name, T):
    wl = W.WORKLOADS[name].scaled(T)
    routes = torch.from_numpy(np.array(W.make_routes(wl))).to(DEV)
    q, k, v, do = (x.to(DEV) for x in W.make_tensors(wl))
    return wl, routes, q, k, v, do


@pytest.mark.parametrize("name,T", [("tiny", 256), ("seq4k", 1024), ("thd16k", 2048), ("seq32k", 1024),
                                    ("cp128k", 256)])
@pytest.mark.parametrize("kv_fp32", [False, True])
def test_saved_rows_backward_equals_sorting_backward(name, T, kv_fp32):
    wl, routes, q, k, v, do = _inputs(name, T)
    H, G, n_sel = wl.H, wl.G, routes.shape[1]
    fws = torch.empty(qsa.forward_workspace_size(T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    out, lse = qsa.forward(q, k, v, routes, wl.scale, workspace=fws)
    ref = qsa.backward(do, q, k, v, out, lse, routes, wl.scale, kv_fp32=kv_fp32)
    got = qsa.backward(do, q, k, v, out, lse, routes, wl.scale, kv_fp32=kv_fp32, saved_workspace=fws)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_saved_rows_in_the_backward_workspace_itself():
    wl, routes, q, k, v, do = _inputs("thd16k", 1024)
    H, G, n_sel = wl.H, wl.G, routes.shape[1]
    ws = torch.empty(qsa.backward_workspace_size(wl.T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    out, lse = qsa.forward(q, k, v, routes, wl.scale)
    ref = qsa.backward(do, q, k, v, out, lse, routes, wl.scale)
    out2, lse2 = qsa.forward(q, k, v, routes, wl.scale, workspace=ws)
    got = qsa.backward(do, q, k, v, out2, lse2, routes, wl.scale, workspace=ws, saved_workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, out) and torch.equal(lse2, lse)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    assert int(ws[:4].view(torch.int32).item()) == 0  # status word: no wait gave up


def test_saved_rows_without_a_forward_report_a_bad_status():
    # a forward workspace that no forward wrote (zero-filled here, so that even
    # an unguarded read would see empty rows) lacks the route-list tag: the
    # status word reports it and no kernel reads the lists
    wl, routes, q, k, v, do = _inputs("thd16k", 1024)
    H, G, n_sel = wl.H, wl.G, routes.shape[1]
    out, lse = qsa.forward(q, k, v, routes, wl.scale)
    fws = torch.zeros(qsa.forward_workspace_size(wl.T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    ws = torch.empty(qsa.backward_workspace_size(wl.T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    qsa.backward(do, q, k, v, out, lse, routes, wl.scale, workspace=ws, saved_workspace=fws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 2
    # a forward on the same buffer writes the tag: the same call then succeeds
    qsa.forward(q, k, v, routes, wl.scale, workspace=fws)
    ref = qsa.backward(do, q, k, v, out, lse, routes, wl.scale)
    got = qsa.backward(do, q, k, v, out, lse, routes, wl.scale, workspace=ws, saved_workspace=fws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
