"""No kernel writes outside its outputs or its workspace.

Every output and the workspace are views into larger buffers whose margins hold
a fixed byte pattern; after forward + backward the margins must be unchanged."""
import numpy as np
import pytest
import torch

from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
GUARD = 4096          # bytes of margin on each side (keeps 256-byte alignment)
PATTERN = 0xA5


def _guarded(shape, dtype):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device=DEV)
    view = raw[GUARD:GUARD + n].view(dtype).view(shape)
    return raw, view


def _margins_intact(raw):
    head, tail = raw[:GUARD], raw[-GUARD:]
    return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


@pytest.mark.parametrize("name,T", [("tiny", None), ("seq32k", 300), ("cp128k", 200)])
def test_no_write_outside_outputs_and_workspace(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].scaled(T)
    routes = torch.from_numpy(np.array(W.make_routes(wl))).to(DEV)
    q, k, v, do = (x.to(DEV) for x in W.make_tensors(wl))
    n_sel = routes.shape[1]
    raws = {}
    raws["out"], out = _guarded(q.shape, torch.bfloat16)
    raws["lse"], lse = _guarded((wl.T, wl.H), torch.float32)
    raws["dq"], dq = _guarded(q.shape, torch.bfloat16)
    raws["dk"], dk = _guarded(k.shape, torch.bfloat16)
    raws["dv"], dv = _guarded(v.shape, torch.bfloat16)
    raws["wsf"], wsf = _guarded((qsa.forward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, n_sel),), torch.uint8)
    raws["wsb"], wsb = _guarded((qsa.backward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, n_sel),), torch.uint8)
    qsa.forward(q, k, v, routes, wl.scale, out=out, lse=lse, workspace=wsf)
    qsa.backward(do, q, k, v, out, lse, routes, wl.scale, dq=dq, dk=dk, dv=dv, workspace=wsb)
    torch.cuda.synchronize()
    for key, raw in raws.items():
        assert _margins_intact(raw), key
    assert torch.isfinite(out.float()).all() and torch.isfinite(dk.float()).all()
