"""GPU parity of the bitmap -> route IDs adapter (``qsa_bitmap_routes``).

The adapter follows the block lookup of the cuDNN-Frontend "Query Sparse
Attention (QSA)" page ("Selection and components"); the oracle is
``oracle.qsa_bitmap``.  Index work: compared bit for bit.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import backward_dense, forward_dense
from oracle.qsa_bitmap import bitmap_route_rows, bitmap_routes
from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda:0"


def _dev(case):
    return {k: torch.from_numpy(np.ascontiguousarray(case[k])).to(DEV)
            for k in ("sel_blocks", "lo", "hi", "blk_base", "tok_base")}


def _run(case, n_sel, block_size=4):
    d = _dev(case)
    routes, cnt, mx = qsa.bitmap_routes(d["sel_blocks"], d["lo"], d["hi"], d["blk_base"], d["tok_base"],
                                        case["T_kv"], n_sel, block_size)
    torch.cuda.synchronize()
    return routes.cpu().numpy(), cnt.cpu().numpy(), int(mx.item())


def test_hand_worked_example():
    fx = json.load(open(os.path.join(HERE, "golden", "bitmap_example.json")))
    case = {k: np.array(fx[k], dtype=np.uint8 if k == "sel_blocks" else np.int32)
            for k in ("sel_blocks", "lo", "hi", "blk_base", "tok_base")}
    case["T_kv"] = fx["T_kv"]
    routes, cnt, mx = _run(case, n_sel=12)
    for t in range(fx["T"]):
        exp = fx["expected_rows"][str(t)]
        assert routes[t].tolist() == exp + [-1] * (12 - len(exp)), t
        assert cnt[t] == len(exp)
    assert mx == max(len(v) for v in fx["expected_rows"].values())


@pytest.mark.parametrize("T,n_docs,blocks,seed", [(1000, 5, 64, 1), (2048, 1, 128, 2), (1537, 9, 300, 3)])
def test_packed_random_bitexact(T, n_docs, blocks, seed):
    case = W.make_bitmap_case(T, n_docs, blocks, seed)
    o_routes, o_cnt = bitmap_routes(case["sel_blocks"], case["lo"], case["hi"], case["blk_base"], case["tok_base"],
                                    case["T_kv"], width=4 * blocks + 8)
    routes, cnt, mx = _run(case, n_sel=4 * blocks + 8)
    assert np.array_equal(routes, o_routes)
    assert np.array_equal(cnt, o_cnt)
    assert mx == int(o_cnt.max())


def test_truncated_rows_keep_smallest_keys_and_true_counts():
    case = W.make_bitmap_case(777, 3, 200, 7)
    o_routes, o_cnt = bitmap_routes(case["sel_blocks"], case["lo"], case["hi"], case["blk_base"], case["tok_base"],
                                    case["T_kv"], width=37)
    routes, cnt, mx = _run(case, n_sel=37)
    assert (o_cnt > 37).any()
    assert np.array_equal(routes, o_routes) and np.array_equal(cnt, o_cnt) and mx == int(o_cnt.max())


@pytest.mark.parametrize("block_size", [1, 3, 8])
def test_other_block_sizes(block_size):
    case = W.make_bitmap_case(500, 4, 40, 11, block_size=block_size)
    o_routes, o_cnt = bitmap_routes(case["sel_blocks"], case["lo"], case["hi"], case["blk_base"], case["tok_base"],
                                    case["T_kv"], width=40 * block_size + 8, block_size=block_size)
    routes, cnt, _ = _run(case, n_sel=40 * block_size + 8, block_size=block_size)
    assert np.array_equal(routes, o_routes) and np.array_equal(cnt, o_cnt)


def test_bitmap_attention_matches_dense_oracle():
    # bitmap input -> adapter -> route-set forward/backward, against the dense
    # oracle on the oracle's own allowed sets
    T, H, G, d = 384, 12, 1, 256
    case = W.make_bitmap_case(T, 3, 24, 5)
    n_sel = 4 * 24 + 8
    o_routes, _ = bitmap_routes(case["sel_blocks"], case["lo"], case["hi"], case["blk_base"], case["tok_base"],
                                T, width=n_sel)
    g = torch.Generator().manual_seed(4321)
    q, k, v, do = (torch.randn(*s, generator=g).to(torch.bfloat16) for s in
                   ((T, H, d), (T, G, d), (T, G, d), (T, H, d)))
    dd = _dev(case)
    routes, _, _ = qsa.bitmap_routes(dd["sel_blocks"], dd["lo"], dd["hi"], dd["blk_base"], dd["tok_base"], T, n_sel)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    out, lse = qsa.forward(qd, kd, vd, routes, 1 / 16)
    dq, dk, dv = qsa.backward(dod, qd, kd, vd, out, lse, routes, 1 / 16)
    qf, kf, vf, dof = (x.double().numpy() for x in (q, k, v, do))
    o_out, o_lse = forward_dense(qf, kf, vf, o_routes, 1 / 16)
    o_dq, o_dk, o_dv = backward_dense(dof, qf, kf, vf, o_routes, 1 / 16)

    def rel(a, b):
        return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-3))

    assert rel(out.double().cpu().numpy(), o_out) <= 1e-2
    lg, lo_ = lse.cpu().numpy(), o_lse
    fin = np.isfinite(lo_)
    assert np.array_equal(np.isneginf(lg), np.isneginf(lo_))
    assert np.abs(lg[fin] - lo_[fin]).max() <= 1e-3
    for a, b in ((dq, o_dq), (dk, o_dk), (dv, o_dv)):
        assert rel(a.double().cpu().numpy(), b) <= 1e-2


def test_full_size_bitmap_of_seq32k_routes():
    # the seq32k routes' blocks as a single-sequence bitmap (T x NB = 32768 x
    # 8192 bytes): the adapter must return exactly each row's unique valid keys
    wl = W.WORKLOADS["seq32k"]
    r = torch.from_numpy(np.array(W.make_routes(wl))).to(DEV)
    T, T_kv = wl.T, wl.T_kv
    NB = T_kv // 4
    sel = torch.zeros((T, NB), dtype=torch.uint8, device=DEV)
    valid = (r >= 0) & (r < T_kv)
    rows = torch.arange(T, device=DEV).unsqueeze(1).expand_as(r)[valid]
    sel[rows, (r[valid] // 4).long()] = 1
    zero = torch.zeros(T, dtype=torch.int32, device=DEV)
    hi = torch.arange(T, dtype=torch.int32, device=DEV)
    routes, cnt, mx = qsa.bitmap_routes(sel, zero, hi, zero, zero, T_kv, 512)
    torch.cuda.synchronize()
    assert int(mx.item()) <= 512
    rng = np.random.default_rng(99)
    rows_np = W.make_routes(wl)
    routes_c = routes.cpu().numpy()
    for t in rng.choice(T, size=256, replace=False):
        u = np.unique(rows_np[t][(rows_np[t] >= 0) & (rows_np[t] < T_kv)])
        assert routes_c[t, :u.size].tolist() == u.tolist() and (routes_c[t, u.size:] == -1).all(), t
