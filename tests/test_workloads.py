"""The seeded generators produce the route structure each workload states."""

import numpy as np
import pytest

from token_indexed_sparse_b200 import workloads as W


def _doc_start(wl, pos):
    rng = np.random.default_rng(wl.seed)
    starts = W._doc_starts(wl, rng)
    return starts[np.searchsorted(starts, pos, side="right") - 1], starts


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_route_structure(name):
    wl = W.WORKLOADS[name]
    r = W.make_routes(wl)
    assert r.shape == (wl.T, wl.W) and r.dtype == np.int32
    assert W.make_routes(wl) is r                       # cached, deterministic
    pos = wl.q_offset + np.arange(wl.T)
    valid = r >= 0
    assert np.all(r[valid] < wl.T_kv)
    assert np.all(np.where(valid, r, 0) <= pos[:, None]), "routes must be causal"
    empty = ~valid.any(axis=1)
    if wl.pad_tail:
        assert empty[-wl.pad_tail:].all()
    expected_pad = int(np.floor(wl.pad_frac * wl.T)) + wl.pad_tail
    assert empty.sum() == expected_pad
    rng = np.random.default_rng(0)
    for t in rng.choice(np.nonzero(~empty)[0], 64, replace=False):
        p = pos[t]
        doc, starts = _doc_start(wl, p)
        ids = r[t][r[t] >= 0].astype(np.int64)
        uniq = np.unique(ids)
        assert np.all(uniq >= doc), "routes stay inside the query's document"
        blocks = np.unique((uniq - doc) // 4)
        own = (p - doc) // 4
        visible = own + 1
        assert len(blocks) == min(wl.blocks, visible)
        if wl.policy != "uniform":
            assert own in blocks
        # every chosen block is complete, except the own block which ends at p
        for b in blocks:
            lo = doc + 4 * b
            want = np.arange(lo, min(lo + 3, p) + 1)
            assert np.all(np.isin(want, uniq))
        if wl.dup_frac:
            assert len(ids) - len(uniq) == int(np.ceil(wl.dup_frac * len(uniq)))
        else:
            assert len(ids) == len(uniq)
            groups = r[t][: 4 * len(blocks)].reshape(-1, 4)
            for grp in groups:          # four-slot groups: a block, -1 padded at its tail
                v = grp[grp >= 0]
                assert len(v) >= 1 and np.all(np.diff(v) == 1) and (v[0] - doc) % 4 == 0
                assert np.all(grp[len(v):] == -1)
    if name == "seq32k":
        # half of a late row's blocks lie in the most recent 512 blocks
        t = wl.T - 1
        uniq = np.unique(r[t][r[t] >= 0])
        blocks = np.unique(uniq // 4)
        assert np.sum(blocks >= (t // 4) - 511) == 64


def test_tensors_are_seeded_bf16():
    import torch
    wl = W.WORKLOADS["tiny"]
    q, k, v, do = W.make_tensors(wl)
    assert q.dtype == torch.bfloat16 and q.shape == (256, 12, 256)
    assert k.shape == v.shape == (256, 1, 256) and do.shape == q.shape
    q2, *_ = W.make_tensors(wl)
    assert torch.equal(q, q2)
    assert abs(float(q.float().std()) - 1.0) < 0.02


def test_pair_count():
    r = np.array([[3, 3, -1, 1, 9], [-1, -1, -1, -1, -1], [0, 1, 2, 3, 4]])
    assert W.pair_count(r, 4) == 2 + 0 + 4


# the seeded recipes are fixed: their routed-pair counts are the ones the
# design documentation and the benchmark figures quote
PAIRS = {"tiny": 13709, "seq4k": 1010176, "thd16k": 7150250, "seq32k": 16598016, "cp128k": 15927894}


@pytest.mark.parametrize("name", list(PAIRS))
def test_seeded_pair_counts(name):
    wl = W.WORKLOADS[name]
    assert W.pair_count(W.make_routes(wl), wl.T_kv) == PAIRS[name]
