"""qsa_forward + qsa_backward captured in one CUDA graph.

Both calls take caller-owned workspaces, allocate nothing, read no device
value on the host and reset their counters with in-stream memsets, so a
captured step must replay exactly what the eager calls compute, and a replay
must read whatever the captured input buffers hold at replay time.
"""
import numpy as np
import pytest
import torch

from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_graph_replays_equal_eager_calls():
    wl = W.WORKLOADS["seq4k"].scaled(1024)
    routes = torch.from_numpy(np.array(W.make_routes(wl))).to(DEV)
    q, k, v, do = (x.to(DEV) for x in W.make_tensors(wl))
    T, H, G, n_sel = wl.T, wl.H, wl.G, routes.shape[1]
    fws = torch.empty(qsa.forward_workspace_size(T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    bws = torch.empty(qsa.backward_workspace_size(T, wl.T_kv, H, G, n_sel), dtype=torch.uint8, device=DEV)
    out, lse = torch.empty_like(q), torch.empty(T, H, dtype=torch.float32, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    results = (out, lse, dq, dk, dv)

    def step():
        qsa.forward(q, k, v, routes, wl.scale, out=out, lse=lse, workspace=fws)
        qsa.backward(do, q, k, v, out, lse, routes, wl.scale, dq=dq, dk=dk, dv=dv, workspace=bws)

    def eager():
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return [t.clone() for t in results]

    ref = eager()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        for t in results:
            t.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(results, ref):
            assert torch.equal(a, b)

    # new values in the captured input buffers: the replay follows them
    gen = torch.Generator(device="cpu").manual_seed(77)
    do.copy_(torch.randn(do.shape, generator=gen).to(do.dtype))
    q.copy_(torch.randn(q.shape, generator=gen).to(q.dtype))
    routes.copy_(torch.flip(routes, dims=[1]))  # same sets, other slot order
    ref2 = eager()
    assert not torch.equal(ref2[2], ref[2])
    for t in results:
        t.fill_(0)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(results, ref2):
        assert torch.equal(a, b)
    del g
