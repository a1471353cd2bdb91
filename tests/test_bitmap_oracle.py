"""Pins of the bitmap-lookup oracle (CPU only).

The lookup is defined in the cuDNN-Frontend "Query Sparse Attention (QSA)"
page, "Selection and components"; the hand-worked fixture, the route
round trip and the special cases below pin it without reusing its code.
"""

import json
import os

import numpy as np

from oracle.qsa_bitmap import bitmap_membership, bitmap_route_rows, bitmap_routes
from oracle import routes_to_membership
from token_indexed_sparse_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def _fixture():
    return json.load(open(os.path.join(HERE, "golden", "bitmap_example.json")))


def test_hand_worked_packed_example():
    fx = _fixture()
    rows = bitmap_route_rows(np.array(fx["sel_blocks"], dtype=np.uint8), fx["lo"], fx["hi"], fx["blk_base"],
                             fx["tok_base"], fx["T_kv"], fx["block_size"])
    for t in range(fx["T"]):
        assert rows[t].tolist() == fx["expected_rows"][str(t)], (t, fx["notes"].get(str(t)))


def test_floor_division_distinguishes_truncation():
    # one row, key 8 two tokens before tok_base 10: floor(-2/4) = -1, truncation 0
    sel = np.zeros((1, 4), np.uint8)
    sel[0, 1] = 1                       # block blk_base - 1 = 1
    A = bitmap_membership(sel, [8], [9], [2], [10], 12, 4)
    assert np.flatnonzero(A[0]).tolist() == [8, 9]
    sel[0] = 0
    sel[0, 2] = 1                       # the block truncation would pick
    A = bitmap_membership(sel, [8], [9], [2], [10], 12, 4)
    assert not A.any()


def _block_routes_to_bitmap(routes, T_kv, block_size=4):
    """Single-sequence bitmap selecting every block that a route row touches."""
    T = routes.shape[0]
    NB = (T_kv + block_size - 1) // block_size
    sel = np.zeros((T, NB), np.uint8)
    for t in range(T):
        r = routes[t]
        r = r[(r >= 0) & (r < T_kv)]
        sel[t, r // block_size] = 1
    return sel


def test_round_trip_of_causal_block_routes():
    # routes made of whole causal four-token blocks plus the causal tail, as the
    # workload recipe draws them: the bitmap of their blocks with bounds
    # [0, t] allows exactly the routed keys
    for wl in (W.WORKLOADS["tiny"], W.WORKLOADS["seq4k"].scaled(256)):
        routes = W.make_routes(wl)
        T, T_kv = routes.shape[0], wl.T_kv
        sel = _block_routes_to_bitmap(routes, T_kv)
        t = np.arange(T)
        A = bitmap_membership(sel, np.zeros(T, int), t + wl.q_offset, np.zeros(T, int), np.zeros(T, int), T_kv)
        M = routes_to_membership(routes, T_kv)
        assert np.array_equal(A, M)


def test_empty_and_out_of_range():
    sel = np.ones((3, 2), np.uint8)
    # row 0: lo > hi; row 1: bounds beyond the key range; row 2: blocks beyond NB
    A = bitmap_membership(sel, [5, 40, 0], [4, 50, 15], [0, 0, 0], [0, 0, 0], 16, 4)
    assert not A[0].any() and not A[1].any()
    assert np.flatnonzero(A[2]).tolist() == list(range(8))   # blocks 0, 1 only (NB = 2)


def test_width_truncation_reports_true_counts():
    sel = np.ones((1, 4), np.uint8)
    routes, counts = bitmap_routes(sel, [0], [15], [0], [0], 16, width=6)
    assert counts.tolist() == [16]
    assert routes[0].tolist() == [0, 1, 2, 3, 4, 5]
