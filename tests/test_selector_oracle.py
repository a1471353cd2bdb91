"""Pins of the selector oracle (CPU only).

The selector is defined on the cuDNN-Frontend "Query Sparse Attention (QSA)"
page ("Finding QSA attention and its indexer") and the route format on the
"cudnn_qsa" page (``_pack_indices``).  The pins below check the oracle against
a hand-worked example, a special case that reduces to a plain sort, algebraic
properties of the score and the route-format invariants.
"""

import json
import os

import numpy as np

from oracle.qsa_selector import n_candidates, own_blocks, select, selector_scores, topk_blocks

HERE = os.path.dirname(os.path.abspath(__file__))


def test_hand_worked_example():
    fx = json.load(open(os.path.join(HERE, "golden", "selector_example.json")))
    S, blocks, routes = select(np.array(fx["qi"]), np.array(fx["kbar"]), fx["scale"], fx["k"])
    for t, v in fx["expected_scores"].items():
        assert np.allclose(S[int(t), :len(v)], v, rtol=0, atol=1e-15), t
    for t, v in fx["expected_blocks"].items():
        assert blocks[int(t)].tolist() == v, (t, fx["notes"].get(t))
    for t, v in fx["expected_routes"].items():
        assert routes[int(t)].tolist() == v, (t, fx["notes"].get(t))


def test_one_head_identity_keys_reduce_to_a_sort():
    # Hi = 1 and kbar = identity: S[t, c] = scale * max(qi[t, 0, c], 0); the
    # top-k is then the k largest entries, equal ones by the lower index
    rng = np.random.default_rng(3)
    T, NB, k = 64, 16, 5
    qi = rng.integers(-3, 4, size=(T, 1, NB)).astype(float)     # many ties
    S = selector_scores(qi, np.eye(NB), 2.0)
    n = n_candidates(T, NB)
    blocks = topk_blocks(S, n, k)
    for t in range(T):
        m = int(n[t])
        r = 2.0 * np.maximum(qi[t, 0, :m], 0)
        exp = np.sort(np.argsort(-r, kind="stable")[:k])
        assert blocks[t, :exp.size].tolist() == exp.tolist() and (blocks[t, exp.size:] == -1).all()


def test_score_homogeneity_and_head_additivity():
    rng = np.random.default_rng(5)
    qi = rng.standard_normal((40, 6, 8))
    kbar = rng.standard_normal((10, 8))
    S = selector_scores(qi, kbar, 0.25)
    S2 = selector_scores(3.0 * qi, kbar, 0.25)
    fin = np.isfinite(S)
    assert np.allclose(S2[fin], 3.0 * S[fin])
    Sa = selector_scores(qi[:, :2], kbar, 0.25)
    Sb = selector_scores(qi[:, 2:], kbar, 0.25)
    assert np.allclose((Sa + Sb)[fin], S[fin])
    # a head whose dot products are all negative adds nothing
    neg = -np.abs(rng.standard_normal((40, 1, 8)))
    kpos = np.abs(kbar)
    assert np.allclose(selector_scores(np.concatenate([np.abs(qi), neg], 1), kpos, 1.0)[fin],
                       selector_scores(np.abs(qi), kpos, 1.0)[fin])


def test_ratio_causal_candidates():
    # huge scores on the own block and later blocks must never be selected
    T, NB, k = 48, 12, 3
    kbar = np.eye(NB)
    qi = np.zeros((T, 1, NB))
    for t in range(T):
        qi[t, 0, t // 4:] = 1e6          # own block and later
        qi[t, 0, : t // 4] = np.arange(t // 4)
    _, blocks, routes = select(qi, kbar, 1.0, k)
    for t in range(T):
        sel = blocks[t][blocks[t] >= 0]
        assert (sel < t // 4).all() and sel.size == min(k, t // 4)
        assert set(range(4 * (t // 4), t + 1)) <= set(routes[t].tolist())   # the causal tail


def test_packed_sequences_and_route_format():
    rng = np.random.default_rng(9)
    # two documents: tokens 0..13 and 14..40 (origin 14 is not a multiple of 4)
    T = 41
    tok_base = np.where(np.arange(T) < 14, 0, 14)
    blk_base = np.where(np.arange(T) < 14, 0, 4)        # document A has blocks 0..3
    NB = 4 + 7
    qi = rng.standard_normal((T, 3, 4))
    kbar = rng.standard_normal((NB, 4))
    k = 3
    S, blocks, routes = select(qi, kbar, 0.5, k, blk_base=blk_base, tok_base=tok_base)
    for t in range(T):
        local = t - tok_base[t]
        own = local // 4
        # scores use the document's own compressed blocks
        for c in range(own):
            exp = 0.5 * np.maximum(qi[t] @ kbar[blk_base[t] + c], 0).sum()
            assert abs(S[t, c] - exp) < 1e-12
        row = routes[t]
        groups = row.reshape(-1, 4)
        seen = []
        for gidx, grp in enumerate(groups):
            v = grp[grp >= 0]
            if v.size == 0:
                assert (grp == -1).all()
                continue
            assert (np.diff(v) == 1).all()                    # consecutive tokens
            assert (grp[:v.size] == v).all()                  # -1 only at the end
            start = v[0] - tok_base[t]
            assert start % 4 == 0                             # block-aligned in the document
            if v.size < 4 or start // 4 == own:
                assert start // 4 == own and v[-1] == t       # the causal tail
            seen.extend(v.tolist())
        assert seen == sorted(set(seen))                      # distinct, ascending


def test_candidates_stop_at_the_last_compressed_block():
    # 40 queries but only 6 compressed blocks: later queries see blocks 0..5
    T, NB = 40, 6
    assert n_candidates(T, NB).tolist() == [min(t // 4, NB) for t in range(T)]
    assert own_blocks(T).tolist() == [t // 4 for t in range(T)]
    rng = np.random.default_rng(2)
    S, blocks, routes = select(rng.standard_normal((T, 2, 4)), rng.standard_normal((NB, 4)), 1.0, 8)
    assert (blocks[39][blocks[39] >= 0] < NB).all() and (blocks[39] >= 0).sum() == NB
    assert routes[39].tolist()[4 * NB:4 * NB + 4] == [36, 37, 38, 39]
