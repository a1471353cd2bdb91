"""Plain FP64 CPU restatement of exact route-set Query Sparse Attention (QSA).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA product path.

Sources (documentation pages, cited by page title and section):

* [FLEX] "nemo_automodel.components.models.qwen3_8_flash_next.flex_qsa",
  module description (each query row attends exactly to its route IDs; rows
  whose routes are all -1 give zero output and zero gradients) and
  ``_routes_to_membership`` (scatter of route IDs into a boolean
  ``[B, S_q, kv_length]`` table; negative or out-of-range entries are padding).
* [FA4] "nemo_automodel.components.models.qwen3_8_flash_next.fa4_qsa",
  ``_preprocess`` (duplicate IDs collapse, invalid IDs are discarded; forward
  and reverse block lists) and ``fa4_sparse_gqa_attention`` (duplicates select
  a token once, empty rows have zero output and query gradients, no implicit
  triangular mask, query heads a positive multiple of KV heads).
* [CUDNN] "nemo_automodel.components.models.qwen3_8_flash_next.cudnn_qsa",
  ``_CudnnQSA`` (one independent GQA head group per KV head).
* [QSA] cuDNN-Frontend "Query Sparse Attention (QSA)": section "Tensors"
  (LSE is the natural-log softmax normaliser; dK/dV are summed over query
  heads) and section "Selection and components" (forward: scaled QK, softmax,
  PV; empty rows give zero output and -inf LSE; the backward equations
  S, P, delta, dP, dS, dQ, dK, dV).

Readings where the pages leave a step open:

* Query head ``h`` uses KV head ``h // (H // G)`` (contiguous head groups).
* ``delta`` is formed from the oracle's own exact output.
* A route ID ``r`` is valid iff ``0 <= r < kv_length``; everything else is padding.

Array conventions: ``q``/``grad_out``/``out``/``dq`` are ``[T, H, D]``;
``k``/``v``/``dk``/``dv`` are ``[T_kv, G, D]``; ``routes`` is ``[T, W]`` of
integers; ``lse`` is ``[T, H]``.  Everything is computed in float64.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _head_groups(H: int, G: int) -> int:
    if G <= 0 or H <= 0 or H % G != 0:
        raise ValueError("query heads must be a positive multiple of KV heads")
    return H // G


# ---------------------------------------------------------------------------
# Route sets
# ---------------------------------------------------------------------------

def routes_to_membership(routes, kv_length: int) -> np.ndarray:
    """Boolean membership table ``M[t, j]`` = "query t routes to key j".

    [FLEX] ``_routes_to_membership``: route IDs are scattered into a boolean
    table; negative and out-of-range IDs are padding.  Scattering into a
    boolean table makes duplicates collapse ([FA4] ``_preprocess``).
    """
    r = np.asarray(routes).astype(np.int64)
    T, W = r.shape
    M = np.zeros((T, kv_length), dtype=bool)
    valid = (r >= 0) & (r < kv_length)
    rows = np.broadcast_to(np.arange(T)[:, None], (T, W))
    M[rows[valid], r[valid]] = True
    return M


def row_route_sets(routes, kv_length: int) -> list:
    """Per query row, the sorted set of valid route IDs (the set R_t)."""
    r = np.asarray(routes).astype(np.int64)
    out = []
    for row in r:
        keep = row[(row >= 0) & (row < kv_length)]
        out.append(np.unique(keep))
    return out


def route_rows_csr(routes, kv_length: int):
    """Row-wise sorted, de-duplicated valid route IDs.

    Returns ``(counts [T] int32, cols [T, W] int32)``; row ``t`` holds its
    ``counts[t]`` IDs ascending in ``cols[t, :counts[t]]`` and -1 after them.
    This is the set R_t of [FA4] ``_preprocess`` written out per row.
    """
    r = np.asarray(routes)
    T, W = r.shape
    counts = np.zeros(T, dtype=np.int32)
    cols = np.full((T, W), -1, dtype=np.int32)
    for t, s in enumerate(row_route_sets(r, kv_length)):
        counts[t] = len(s)
        cols[t, : len(s)] = s
    return counts, cols


def key_quad_lists(routes, kv_length: int):
    """Key -> query transpose of the route sets, grouped by aligned key quads.

    The reverse lists of [FA4] ``_preprocess`` at a granularity of four keys:
    quad ``b`` covers keys ``4b .. 4b+3``.  For each quad, the queries whose
    route set meets the quad are listed in ascending order, each with a 4-bit
    owner mask (bit ``i`` set iff key ``4b+i`` is in that query's set).

    Returns ``(quad_ptr [n_quads+1] int64, quad_query [E] int32,
    quad_mask [E] int32)`` with ``n_quads = ceil(kv_length / 4)``.
    """
    n_quads = (kv_length + 3) // 4
    per_quad = [dict() for _ in range(n_quads)]
    for t, s in enumerate(row_route_sets(routes, kv_length)):
        for j in s:
            b = int(j) >> 2
            per_quad[b][t] = per_quad[b].get(t, 0) | (1 << (int(j) & 3))
    ptr = np.zeros(n_quads + 1, dtype=np.int64)
    qs, ms = [], []
    for b in range(n_quads):
        items = sorted(per_quad[b].items())
        ptr[b + 1] = ptr[b] + len(items)
        qs.extend(t for t, _ in items)
        ms.extend(m for _, m in items)
    return ptr, np.asarray(qs, dtype=np.int32), np.asarray(ms, dtype=np.int32)



def key_tile_lists(routes, kv_length: int, tile: int = 128):
    """Key -> query transpose of the route sets, grouped by aligned key tiles.

    The reverse lists of [FA4] ``_preprocess`` at a granularity of ``tile``
    keys: tile ``b`` covers keys ``tile*b .. tile*b + tile - 1``.  For each
    tile, the queries whose route set meets it are listed in ascending order,
    each with ``i0`` = the number of keys of R_t below the tile (the position of
    its first key in the sorted row) and ``n`` = the number of keys of R_t in
    the tile.

    Returns ``(tile_ptr [n_tiles+1] int64, query [E] int32, i0 [E] int32,
    n [E] int32)`` with ``n_tiles = ceil(kv_length / tile)``.
    """
    n_tiles = (kv_length + tile - 1) // tile
    per_tile = [[] for _ in range(n_tiles)]
    for t, s in enumerate(row_route_sets(routes, kv_length)):
        tiles = s // tile
        for b in np.unique(tiles):
            pos = np.nonzero(tiles == b)[0]
            per_tile[int(b)].append((t, int(pos[0]), int(pos.size)))
    ptr = np.zeros(n_tiles + 1, dtype=np.int64)
    for b in range(n_tiles):
        ptr[b + 1] = ptr[b] + len(per_tile[b])
    flat = [e for lst in per_tile for e in lst]   # rows were visited in ascending t
    cols = np.asarray(flat, dtype=np.int32).reshape(-1, 3)
    return ptr, cols[:, 0].copy(), cols[:, 1].copy(), cols[:, 2].copy()

def query_union_lists(routes, kv_length: int, group: int):
    """Route sets of adjacent query rows merged, with owner masks.

    The paired-query gather of the [QSA] page ("Selection and components": one
    program owns adjacent queries and gathers the union of their selected
    blocks once, with owner bits telling which query selected each) at a group
    of ``group`` consecutive rows: group ``i`` holds rows ``group*i ..
    group*i + group - 1`` (the last group may be shorter).  Its list is the
    union of those rows' route sets R_t in ascending key order, and key j's
    owner mask has bit ``q`` set iff j is in R_{group*i + q}.

    Returns ``(counts [n_groups] int32, keys list of int32 arrays, owners list
    of int32 arrays)``, one array pair per group.
    """
    sets = row_route_sets(routes, kv_length)
    T = len(sets)
    n_groups = (T + group - 1) // group
    counts = np.zeros(n_groups, dtype=np.int32)
    keys, owners = [], []
    for i in range(n_groups):
        own = {}
        for q in range(group):
            t = group * i + q
            if t >= T:
                break
            for j in sets[t]:
                own[int(j)] = own.get(int(j), 0) | (1 << q)
        ks = sorted(own)
        counts[i] = len(ks)
        keys.append(np.asarray(ks, dtype=np.int32))
        owners.append(np.asarray([own[j] for j in ks], dtype=np.int32))
    return counts, keys, owners


# ---------------------------------------------------------------------------
# Dense-table form: the definition, for finite inputs
# ---------------------------------------------------------------------------

def _masked_softmax(S: np.ndarray, M: np.ndarray):
    """Row softmax of ``S`` restricted to ``M``; returns (P, lse).

    [QSA] "Selection and components": LSE is the natural-log normaliser and an
    empty row has LSE = -inf and contributes nothing.
    """
    nonempty = M.any(axis=1)
    Sm = np.where(M, S, -np.inf)
    m = np.where(nonempty, Sm.max(axis=1, initial=-np.inf), 0.0)
    E = np.where(M, np.exp(np.where(M, S, 0.0) - m[:, None]), 0.0)
    l = E.sum(axis=1)
    lse = np.where(nonempty, m + np.log(np.where(nonempty, l, 1.0)), -np.inf)
    P = E / np.where(nonempty, l, 1.0)[:, None]
    return P, lse


def forward_dense(q, k, v, routes, scale: float):
    """out, lse by masked dense attention over the membership table.

    [QSA] "Selection and components", forward: S = scale * Q K^T restricted to
    the routed keys, softmax, P V.  No causal mask is added ([FA4]
    ``fa4_sparse_gqa_attention``).  Query head h reads KV head h // (H/G).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = _head_groups(H, G)
    M = routes_to_membership(routes, T_kv)
    out = np.zeros((T, H, D))
    lse = np.zeros((T, H))
    for h in range(H):
        g = h // hpg
        S = scale * (q[:, h, :] @ k[:, g, :].T)
        P, lse[:, h] = _masked_softmax(S, M)
        out[:, h, :] = P @ v[:, g, :]
    return out, lse


def backward_dense(grad_out, q, k, v, routes, scale: float):
    """dq, dk, dv by the backward equations over the dense table.

    [QSA] "Selection and components", backward equations, per query head and
    its KV head: P = exp(S - lse) (zero outside the routed keys),
    delta = rowsum(dO * out), dP = dO V^T, dS = P * (dP - delta),
    dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO; dK/dV summed over the
    query heads that share a KV head ([QSA] "Tensors").
    """
    do, q, k, v = _f64(grad_out), _f64(q), _f64(k), _f64(v)
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = _head_groups(H, G)
    M = routes_to_membership(routes, T_kv)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(H):
        g = h // hpg
        S = scale * (q[:, h, :] @ k[:, g, :].T)
        P, _ = _masked_softmax(S, M)
        out_h = P @ v[:, g, :]
        delta = (do[:, h, :] * out_h).sum(axis=1)
        dP = do[:, h, :] @ v[:, g, :].T
        dS = P * (dP - delta[:, None])
        dq[:, h, :] = scale * (dS @ k[:, g, :])
        dk[:, g, :] += scale * (dS.T @ q[:, h, :])
        dv[:, g, :] += P.T @ do[:, h, :]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Row-gather form: same formulas, one query row at a time over R_t only
# ---------------------------------------------------------------------------

def _row_group(qh, Kg, Vg, scale):
    """Softmax attention of one query's heads ``qh [h, D]`` over gathered keys."""
    S = scale * (qh @ Kg.T)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    P = E / l[:, None]
    return P, m + np.log(l), P @ Vg


def forward_rows(q, k, v, routes, scale: float, rows=None):
    """out, lse for the listed query rows, touching only routed K/V rows.

    Same definition as :func:`forward_dense`, evaluated per row on the gathered
    set R_t, so unselected K/V rows are never read (the isolation that [QSA]
    "Selection and components" requires for non-finite K/V).
    Returns ``out [n, H, D]`` and ``lse [n, H]`` for ``rows`` (default: all).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = _head_groups(H, G)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    sets = row_route_sets(np.asarray(routes)[rows], T_kv)
    out = np.zeros((len(rows), H, D))
    lse = np.full((len(rows), H), -np.inf)
    for i, (t, R) in enumerate(zip(rows, sets)):
        if len(R) == 0:
            continue
        for g in range(G):
            hs = slice(g * hpg, (g + 1) * hpg)
            _, lse[i, hs], out[i, hs, :] = _row_group(q[t, hs, :], k[R, g, :], v[R, g, :], scale)
    return out, lse


def _row_backward(dq_h, qh, Kg, Vg, scale):
    P, _, o = _row_group(qh, Kg, Vg, scale)
    delta = (dq_h * o).sum(axis=1)
    dP = dq_h @ Vg.T
    dS = P * (dP - delta[:, None])
    return P, dS


def backward_rows(grad_out, q, k, v, routes, scale: float, rows=None):
    """dq for the listed rows, and dk/dv accumulated from those rows only.

    The backward equations of [QSA] "Selection and components", one query row
    and one KV group at a time over the gathered set R_t.  With ``rows=None``
    (all rows) dk/dv are the full gradients.
    """
    do, q, k, v = _f64(grad_out), _f64(q), _f64(k), _f64(v)
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = _head_groups(H, G)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    sets = row_route_sets(np.asarray(routes)[rows], T_kv)
    dq = np.zeros((len(rows), H, D))
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for i, (t, R) in enumerate(zip(rows, sets)):
        if len(R) == 0:
            continue
        for g in range(G):
            hs = slice(g * hpg, (g + 1) * hpg)
            Kg, Vg = k[R, g, :], v[R, g, :]
            P, dS = _row_backward(do[t, hs, :], q[t, hs, :], Kg, Vg, scale)
            dq[i, hs, :] = scale * (dS @ Kg)
            dk[R, g, :] += scale * (dS.T @ q[t, hs, :])
            dv[R, g, :] += P.T @ do[t, hs, :]
    return dq, dk, dv


def backward_keys(grad_out, q, k, v, routes, scale: float, keys):
    """Exact dk/dv at the listed key rows (all groups), from every query.

    Finds every query whose route set contains one of ``keys``, evaluates that
    query's full row (its softmax normaliser and delta need all of R_t), and
    keeps the contributions that land on ``keys``.  Returns
    ``(dk [n, G, D], dv [n, G, D])``.
    """
    do, q, k, v = _f64(grad_out), _f64(q), _f64(k), _f64(v)
    T, H, D = q.shape
    T_kv, G, _ = k.shape
    hpg = _head_groups(H, G)
    keys = np.asarray(keys, dtype=np.int64)
    pos = {int(j): n for n, j in enumerate(keys)}
    dk = np.zeros((len(keys), G, D))
    dv = np.zeros((len(keys), G, D))
    r = np.asarray(routes).astype(np.int64)
    hit = np.isin(r, keys).any(axis=1)
    for t in np.nonzero(hit)[0]:
        R = row_route_sets(r[t : t + 1], T_kv)[0]
        sel = [n for n, j in enumerate(R) if int(j) in pos]
        if not sel:
            continue
        for g in range(G):
            hs = slice(g * hpg, (g + 1) * hpg)
            Kg, Vg = k[R, g, :], v[R, g, :]
            P, dS = _row_backward(do[t, hs, :], q[t, hs, :], Kg, Vg, scale)
            for n in sel:
                dst = pos[int(R[n])]
                dk[dst, g, :] += scale * (dS[:, n] @ q[t, hs, :])
                dv[dst, g, :] += P[:, n] @ do[t, hs, :]
    return dk, dv
