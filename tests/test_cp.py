"""Context-parallel plumbing on CPU processes (gloo, world sizes 2 and 4).

The CP path (``token_indexed_sparse_b200.cp``) gathers K/V, runs the local
attention of each rank's query rows and reduce-scatters the dK/dV partials.
Here the local attention is the FP64 oracle, so the test checks the
composition: the ranks' results put together must equal the single-process
oracle on all rows (the "flex_qsa" page: context parallelism is local queries
against gathered global K/V, and reduces to each row attending to its routes).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from token_indexed_sparse_b200 import cp
from token_indexed_sparse_b200 import workloads as W


def test_balanced_query_ranges():
    rng = np.random.default_rng(1)
    counts = rng.integers(0, 50, size=1000)
    for world in (1, 2, 3, 8):
        r = cp.balanced_query_ranges(counts, world)
        assert r[0][0] == 0 and r[-1][1] == 1000
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        per = [counts[s:e].sum() for s, e in r]
        assert max(per) - min(per) <= 2 * counts.max()
    # all rows empty: the ranges still cover every row exactly once
    assert sum(e - s for s, e in cp.balanced_query_ranges([0, 0, 0], 2)) == 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    wl = W.WORKLOADS["seq4k"].scaled(256)          # T = T_kv = 256, 12Q/1KV
    routes = np.array(W.make_routes(wl))
    q, k, v, do = (x.double() for x in W.make_tensors(wl))
    return wl, routes, q, k, v, do


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import backward_dense, forward_dense
        wl, routes, q, k, v, do = _case()
        counts = [(np.unique(r[(r >= 0) & (r < wl.T_kv)])).size for r in routes]
        s, e = cp.balanced_query_ranges(counts, world)[rank]
        ks, ke = cp.kv_slice(wl.T_kv, world, rank)

        def fwd(q_, k_, v_, r_, sc):
            o, l = forward_dense(q_.numpy(), k_.numpy(), v_.numpy(), r_.numpy(), sc)
            return torch.from_numpy(o), torch.from_numpy(l)

        def bwd(go, q_, k_, v_, o_, l_, r_, sc):
            return tuple(torch.from_numpy(x) for x in
                         backward_dense(go.numpy(), q_.numpy(), k_.numpy(), v_.numpy(), r_.numpy(), sc))

        rl = torch.from_numpy(routes[s:e])
        out, lse = cp.cp_forward(q[s:e], k[ks:ke], v[ks:ke], rl, wl.scale, local_forward=fwd)
        # FP64 partials from the oracle, summed across ranks and kept in FP64 (no final rounding)
        dq, dk, dv = cp.cp_backward(do[s:e], q[s:e], k[ks:ke], v[ks:ke], out, lse, rl, wl.scale, local_backward=bwd,
                                    final_cast=lambda x: x)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), s=s, e=e, ks=ks, ke=ke, out=out.numpy(),
                 lse=lse.numpy(), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_cp_composition_matches_single_process(tmp_path, world):
    from oracle import backward_dense, forward_dense
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    wl, routes, q, k, v, do = _case()
    o, l = forward_dense(q.numpy(), k.numpy(), v.numpy(), routes, wl.scale)
    dq, dk, dv = backward_dense(do.numpy(), q.numpy(), k.numpy(), v.numpy(), routes, wl.scale)
    covered_q, covered_k = 0, 0
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        s, e, ks, ke = int(z["s"]), int(z["e"]), int(z["ks"]), int(z["ke"])
        covered_q += e - s
        covered_k += ke - ks
        assert np.allclose(z["out"], o[s:e], rtol=0, atol=1e-12)
        assert np.array_equal(np.isneginf(z["lse"]), np.isneginf(l[s:e]))
        fin = np.isfinite(l[s:e])
        assert np.allclose(z["lse"][fin], l[s:e][fin], rtol=0, atol=1e-12)
        assert np.allclose(z["dq"], dq[s:e], rtol=0, atol=1e-12)
        assert np.allclose(z["dk"], dk[ks:ke], rtol=0, atol=1e-11)
        assert np.allclose(z["dv"], dv[ks:ke], rtol=0, atol=1e-11)
    assert covered_q == wl.T and covered_k == wl.T_kv
