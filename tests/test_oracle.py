"""Pins for the FP64 CPU oracle: each check compares it with something other
than itself (hand-worked values, a brute-force per-pair loop, PyTorch's causal
attention, closed forms, finite differences, invariants)."""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from token_indexed_sparse_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _random_routes(rng, T, T_kv, width, causal=False, q_offset=0):
    r = rng.integers(-3, T_kv + 3, size=(T, width))
    if causal:
        pos = q_offset + np.arange(T)[:, None]
        r = np.where(r <= pos, r, -1)
    return r.astype(np.int64)


# ---------------------------------------------------------------------------
# hand-worked example
# ---------------------------------------------------------------------------

def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    q, k, v, do = (np.array(g[n]) for n in ("q", "k", "v", "grad_out"))
    routes = np.array(g["routes"])
    out, lse = oracle.forward_dense(q, k, v, routes, g["scale"])
    np.testing.assert_allclose(out, g["out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, g["lse"], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, g["scale"])
    np.testing.assert_allclose(dq, g["dq"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk, g["dk"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv, g["dv"], rtol=0, atol=1e-14)
    for fn in (oracle.forward_rows,):
        o2, l2 = fn(q, k, v, routes, g["scale"])
        np.testing.assert_allclose(o2, g["out"], atol=1e-14)
        np.testing.assert_allclose(l2, g["lse"], atol=1e-14)
    dq2, dk2, dv2 = oracle.backward_rows(do, q, k, v, routes, g["scale"])
    np.testing.assert_allclose(dq2, g["dq"], atol=1e-14)
    np.testing.assert_allclose(dk2, g["dk"], atol=1e-14)
    np.testing.assert_allclose(dv2, g["dv"], atol=1e-14)


# ---------------------------------------------------------------------------
# brute-force per-pair loop (independent code, plain Python sums)
# ---------------------------------------------------------------------------

def _brute(q, k, v, do, routes, scale):
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = H // G
    out = np.zeros((T, H, D)); lse = np.full((T, H), -math.inf)
    dq = np.zeros((T, H, D)); dk = np.zeros((T_kv, G, D)); dv = np.zeros((T_kv, G, D))
    for t in range(T):
        R = sorted({int(r) for r in routes[t] if 0 <= r < T_kv})
        if not R:
            continue
        for h in range(H):
            g = h // hpg
            s = {j: scale * sum(q[t, h, d] * k[j, g, d] for d in range(D)) for j in R}
            mx = max(s.values())
            z = sum(math.exp(s[j] - mx) for j in R)
            lse[t, h] = mx + math.log(z)
            p = {j: math.exp(s[j] - lse[t, h]) for j in R}
            for d in range(D):
                out[t, h, d] = sum(p[j] * v[j, g, d] for j in R)
            delta = sum(do[t, h, d] * out[t, h, d] for d in range(D))
            for j in R:
                dp = sum(do[t, h, d] * v[j, g, d] for d in range(D))
                ds = p[j] * (dp - delta)
                for d in range(D):
                    dq[t, h, d] += scale * ds * k[j, g, d]
                    dk[j, g, d] += scale * ds * q[t, h, d]
                    dv[j, g, d] += p[j] * do[t, h, d]
    return out, lse, dq, dk, dv


@pytest.mark.parametrize("T,T_kv,H,G,D", [(24, 24, 4, 2, 16), (10, 14, 12, 1, 24), (6, 9, 6, 3, 8)])
def test_brute_force_pair_loop(T, T_kv, H, G, D):
    rng = np.random.default_rng(T * 100 + D)
    q, do = _rand(rng, T, H, D), _rand(rng, T, H, D)
    k, v = _rand(rng, T_kv, G, D), _rand(rng, T_kv, G, D)
    routes = _random_routes(rng, T, T_kv, 7)
    routes[1] = -1
    ref = _brute(q, k, v, do, routes, 0.3)
    out, lse = oracle.forward_dense(q, k, v, routes, 0.3)
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, 0.3)
    for a, b in zip((out, lse, dq, dk, dv), ref):
        fin = np.isfinite(b)
        assert np.array_equal(np.isfinite(a), fin)
        np.testing.assert_allclose(a[fin], b[fin], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# all-causal routes == ordinary causal attention (PyTorch, float64)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,H,G", [(48, 12, 1), (20, 24, 2)])
def test_causal_routes_equal_causal_attention(T, H, G):
    rng = np.random.default_rng(7 + T)
    D, scale = 256, 1.0 / 16
    q, do = _rand(rng, T, H, D), _rand(rng, T, H, D)
    k, v = _rand(rng, T, G, D), _rand(rng, T, G, D)
    routes = np.where(np.arange(T)[None, :] <= np.arange(T)[:, None], np.arange(T)[None, :], -1)
    routes = routes[:, rng.permutation(T)]          # order inside a row is irrelevant
    out, lse = oracle.forward_dense(q, k, v, routes, scale)
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, scale)

    tq = torch.tensor(q).permute(1, 0, 2)[None].requires_grad_(True)
    tk = torch.tensor(k).permute(1, 0, 2)[None].requires_grad_(True)
    tv = torch.tensor(v).permute(1, 0, 2)[None].requires_grad_(True)
    ke, ve = tk.repeat_interleave(H // G, dim=1), tv.repeat_interleave(H // G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, ke, ve, is_causal=True, scale=scale)
    ref.backward(torch.tensor(do).permute(1, 0, 2)[None])
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).detach().numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)

    # natural-log LSE from PyTorch's CPU flash-attention kernel
    _, ref_lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(
        tq.detach(), ke.detach(), ve.detach(), 0.0, True, scale=scale)[:2]
    np.testing.assert_allclose(lse, ref_lse[0].T.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# padding rows, duplicates, invalid IDs, permutations
# ---------------------------------------------------------------------------

def _case(seed=3, T=12, T_kv=16, H=12, G=1, D=32, width=9):
    rng = np.random.default_rng(seed)
    q, do = _rand(rng, T, H, D), _rand(rng, T, H, D)
    k, v = _rand(rng, T_kv, G, D), _rand(rng, T_kv, G, D)
    routes = _random_routes(rng, T, T_kv, width)
    return rng, q, k, v, do, routes


def test_padding_rows_zero_output_and_gradients():
    rng, q, k, v, do, routes = _case()
    routes[[2, 5]] = -1
    routes[7] = [-1, 16, 99, -7, 2**31 - 1, -1, 17, 16, -2]   # all invalid for T_kv=16
    out, lse = oracle.forward_dense(q, k, v, routes, 0.2)
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, 0.2)
    for t in (2, 5, 7):
        assert np.all(out[t] == 0) and np.all(lse[t] == -np.inf) and np.all(dq[t] == 0)
    do2 = do.copy()
    do2[[2, 5, 7]] = 1e3 * _rand(rng, 3, *do.shape[1:])
    dq2, dk2, dv2 = oracle.backward_dense(do2, q, k, v, routes, 0.2)
    np.testing.assert_array_equal(dk2, dk)
    np.testing.assert_array_equal(dv2, dv)
    np.testing.assert_array_equal(dq2, dq)


def test_duplicates_and_invalid_ids_are_a_set():
    rng, q, k, v, do, routes = _case(seed=5)
    T_kv = k.shape[0]
    clean = np.where((routes >= 0) & (routes < T_kv), routes, -1)
    noisy = np.concatenate([routes, routes[:, ::-1], np.full((routes.shape[0], 3), -5),
                            np.tile([[T_kv, T_kv + 7, 2**40]], (routes.shape[0], 1))], axis=1)
    a = oracle.forward_dense(q, k, v, clean, 0.2)
    b = oracle.forward_dense(q, k, v, noisy, 0.2)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    ga = oracle.backward_dense(do, q, k, v, clean, 0.2)
    gb = oracle.backward_dense(do, q, k, v, noisy, 0.2)
    for x, y in zip(ga, gb):
        np.testing.assert_array_equal(x, y)
    # the row form agrees with the dense form on the noisy routes too
    o2, l2 = oracle.forward_rows(q, k, v, noisy, 0.2)
    np.testing.assert_allclose(o2, b[0], rtol=1e-12, atol=1e-13)


def test_route_order_is_irrelevant():
    rng, q, k, v, do, routes = _case(seed=9)
    perm = np.stack([rng.permutation(routes.shape[1]) for _ in range(routes.shape[0])])
    shuffled = np.take_along_axis(routes, perm, axis=1)
    for x, y in zip(oracle.backward_rows(do, q, k, v, routes, 0.2),
                    oracle.backward_rows(do, q, k, v, shuffled, 0.2)):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-14)


def test_single_route_closed_form():
    rng, q, k, v, do, routes = _case(seed=11, H=24, G=2)
    routes[:] = -1
    routes[4, [0, 3, 8]] = 6          # one route, given three times
    routes[9, 1] = 6
    out, lse = oracle.forward_dense(q, k, v, routes, 0.25)
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, 0.25)
    for t in (4, 9):
        for h in range(24):
            g = h // 12
            np.testing.assert_allclose(out[t, h], v[6, g], atol=1e-14)
            assert abs(lse[t, h] - 0.25 * q[t, h] @ k[6, g]) < 1e-12
        assert np.abs(dq[t]).max() < 1e-13
    for g in range(2):
        hs = slice(12 * g, 12 * g + 12)
        np.testing.assert_allclose(dv[6, g], do[4, hs].sum(0) + do[9, hs].sum(0), atol=1e-12)
        assert np.abs(dk[6, g]).max() < 1e-12
    others = np.ones(k.shape[0], bool); others[6] = False
    assert np.all(dk[others] == 0) and np.all(dv[others] == 0)


def test_all_keys_lse_is_logsumexp():
    from scipy.special import logsumexp
    rng, q, k, v, do, routes = _case(seed=13, T=5, T_kv=7)
    routes = np.tile(np.arange(7), (5, 1))
    _, lse = oracle.forward_dense(q, k, v, routes, 0.5)
    ref = logsumexp(0.5 * np.einsum("thd,jd->thj", q, k[:, 0]), axis=2)
    np.testing.assert_allclose(lse, ref, rtol=1e-13)


# ---------------------------------------------------------------------------
# finite differences of L = sum(dO * out)
# ---------------------------------------------------------------------------

def test_backward_matches_finite_differences():
    rng = np.random.default_rng(17)
    T = T_kv = 16
    H, G, D, scale = 12, 1, 256, 1.0 / 16
    q, do = _rand(rng, T, H, D), _rand(rng, T, H, D)
    k, v = _rand(rng, T_kv, G, D), _rand(rng, T_kv, G, D)
    routes = _random_routes(rng, T, T_kv, 8, causal=True)
    routes[3] = -1
    dq, dk, dv = oracle.backward_dense(do, q, k, v, routes, scale)

    def loss(qq, kk, vv):
        return float((oracle.forward_dense(qq, kk, vv, routes, scale)[0] * do).sum())

    eps = 1e-6
    grads = {"q": (q, dq), "k": (k, dk), "v": (v, dv)}
    for name, (x, gx) in grads.items():
        checks = [rng.standard_normal(x.shape) for _ in range(32)]
        for _ in range(64 // 3 + 1):
            e = np.zeros(x.shape); e.flat[rng.integers(x.size)] = 1.0
            checks.append(e)
        for u in checks:
            args_p = {n: a for n, (a, _) in grads.items()}
            args_m = dict(args_p)
            args_p[name] = x + eps * u
            args_m[name] = x - eps * u
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) -
                  loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * eps)
            an = float((gx * u).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


# ---------------------------------------------------------------------------
# row-gather form == dense form; key-sampled backward == full backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,T", [("tiny", 256), ("seq4k", 256), ("thd16k", 384), ("seq32k", 192),
                                    ("cp128k", 128)])
def test_row_form_matches_dense_form(name, T):
    wl = W.WORKLOADS[name].scaled(T) if T != W.WORKLOADS[name].T else W.WORKLOADS[name]
    routes = W.make_routes(wl)
    rng = np.random.default_rng(wl.seed - 1000)
    q, do = _rand(rng, wl.T, wl.H, 256), _rand(rng, wl.T, wl.H, 256)
    k, v = _rand(rng, wl.T_kv, wl.G, 256), _rand(rng, wl.T_kv, wl.G, 256)
    out_d, lse_d = oracle.forward_dense(q, k, v, routes, wl.scale)
    out_r, lse_r = oracle.forward_rows(q, k, v, routes, wl.scale)
    np.testing.assert_allclose(out_r, out_d, rtol=1e-10, atol=1e-12)
    fin = np.isfinite(lse_d)
    assert np.array_equal(fin, np.isfinite(lse_r))
    np.testing.assert_allclose(lse_r[fin], lse_d[fin], rtol=1e-12)
    gd = oracle.backward_dense(do, q, k, v, routes, wl.scale)
    gr = oracle.backward_rows(do, q, k, v, routes, wl.scale)
    for a, b in zip(gr, gd):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)
    keys = np.unique(rng.integers(0, wl.T_kv, 8))
    dk_s, dv_s = oracle.backward_keys(do, q, k, v, routes, wl.scale, keys)
    np.testing.assert_allclose(dk_s, gd[1][keys], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv_s, gd[2][keys], rtol=1e-9, atol=1e-11)


def test_row_form_isolates_unselected_nonfinite_kv():
    rng, q, k, v, do, routes = _case(seed=21, T_kv=20)
    used = np.unique(routes[(routes >= 0) & (routes < 20)])
    unused = np.setdiff1d(np.arange(20), used)
    assert len(unused) > 0
    k2, v2 = k.copy(), v.copy()
    k2[unused] = np.nan
    v2[unused[::2]] = np.inf
    a = oracle.forward_rows(q, k, v, routes, 0.2)
    b = oracle.forward_rows(q, k2, v2, routes, 0.2)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    ga = oracle.backward_rows(do, q, k, v, routes, 0.2)
    gb = oracle.backward_rows(do, q, k2, v2, routes, 0.2)
    np.testing.assert_array_equal(ga[0], gb[0])
    np.testing.assert_array_equal(ga[1][used], gb[1][used])
    np.testing.assert_array_equal(ga[2][used], gb[2][used])


# ---------------------------------------------------------------------------
# route preprocessing (index work): brute force from the membership table
# ---------------------------------------------------------------------------

def test_route_rows_csr_and_quad_lists():
    rng = np.random.default_rng(23)
    T, T_kv = 40, 37
    routes = _random_routes(rng, T, T_kv, 23)
    routes[5] = -1
    counts, cols = oracle.route_rows_csr(routes, T_kv)
    M = oracle.routes_to_membership(routes, T_kv)
    for t in range(T):
        want = np.nonzero(M[t])[0]
        assert counts[t] == len(want)
        np.testing.assert_array_equal(cols[t, : counts[t]], want)
        assert np.all(cols[t, counts[t]:] == -1)
    ptr, qry, msk = oracle.key_quad_lists(routes, T_kv)
    n_quads = (T_kv + 3) // 4
    assert len(ptr) == n_quads + 1 and ptr[-1] == len(qry) == len(msk)
    for b in range(n_quads):
        entries = []
        for t in range(T):
            m = 0
            for i in range(4):
                if 4 * b + i < T_kv and M[t, 4 * b + i]:
                    m |= 1 << i
            if m:
                entries.append((t, m))
        got = list(zip(qry[ptr[b]:ptr[b + 1]].tolist(), msk[ptr[b]:ptr[b + 1]].tolist()))
        assert got == entries


@pytest.mark.parametrize("tile", [4, 8, 128])
def test_key_tile_lists(tile):
    # brute force from the membership table: the rows meeting each tile, the
    # count of their keys below it and inside it
    rng = np.random.default_rng(29)
    T, T_kv = 45, 301
    routes = _random_routes(rng, T, T_kv, 40)
    routes[7] = -1
    routes[8] = np.arange(40) % 3                      # duplicates inside one tile
    M = oracle.routes_to_membership(routes, T_kv)
    ptr, qry, i0, n = oracle.key_tile_lists(routes, T_kv, tile)
    n_tiles = (T_kv + tile - 1) // tile
    assert len(ptr) == n_tiles + 1 and ptr[-1] == len(qry) == len(i0) == len(n)
    for b in range(n_tiles):
        lo, hi = tile * b, min(T_kv, tile * (b + 1))
        rows = [t for t in range(T) if M[t, lo:hi].any()]
        got = list(zip(qry[ptr[b]:ptr[b + 1]].tolist(), i0[ptr[b]:ptr[b + 1]].tolist(),
                       n[ptr[b]:ptr[b + 1]].tolist()))
        assert got == [(t, int(M[t, :lo].sum()), int(M[t, lo:hi].sum())) for t in rows]


def test_key_tile_lists_refine_quads():
    # tiles of 4 keys are the quads: same rows, and n = popcount of the owner mask
    rng = np.random.default_rng(31)
    routes = _random_routes(rng, 30, 64, 20)
    qptr, qq, qm = oracle.key_quad_lists(routes, 64)
    tptr, tq, _, tn = oracle.key_tile_lists(routes, 64, 4)
    np.testing.assert_array_equal(qptr, tptr)
    np.testing.assert_array_equal(qq, tq)
    np.testing.assert_array_equal([bin(int(m)).count("1") for m in qm], tn)


@pytest.mark.parametrize("group", [1, 2, 4])
def test_query_union_lists(group):
    # brute force from the membership table: per group of adjacent rows, the
    # keys any of them selects (ascending) and, per key, which of them did
    rng = np.random.default_rng(37)
    T, T_kv = 42, 211                                  # the last group is short for group 4
    routes = _random_routes(rng, T, T_kv, 30)
    routes[9] = -1                                     # a padding row inside a group
    routes[10] = routes[11]                            # two rows with the same set
    M = oracle.routes_to_membership(routes, T_kv)
    counts, keys, owners = oracle.query_union_lists(routes, T_kv, group)
    n_groups = (T + group - 1) // group
    assert len(counts) == len(keys) == len(owners) == n_groups
    for i in range(n_groups):
        rows = range(group * i, min(T, group * (i + 1)))
        want = np.nonzero(M[list(rows)].any(axis=0))[0]
        assert counts[i] == len(want)
        np.testing.assert_array_equal(keys[i], want)
        for j, m in zip(keys[i], owners[i]):
            assert m == sum(1 << q for q, t in enumerate(rows) if M[t, j])
    if group == 1:                                     # a group of one row is the row's set
        cnt, cols = oracle.route_rows_csr(routes, T_kv)
        np.testing.assert_array_equal(counts, cnt)
        for t in range(T):
            np.testing.assert_array_equal(keys[t], cols[t, :cnt[t]])
            assert np.all(owners[t] == 1)
