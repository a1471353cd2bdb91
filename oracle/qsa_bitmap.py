"""Plain CPU restatement of the QSA block-selection bitmap lookup.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA product path.

Source: cuDNN-Frontend "Query Sparse Attention (QSA)", section "Tensors"
(``sel_blocks [T, NB]`` uint8, nonzero selects a global block for a query;
``lo``/``hi`` inclusive allowed key-token bounds; ``blk_base`` first global
block and ``tok_base`` first global token of the query's sequence) and section
"Selection and components" (the block lookup: for query t and key token j,
b = blk_base[t] + (j - tok_base[t]) // block_size, and j is allowed iff
lo[t] <= j <= hi[t], 0 <= b < NB and sel_blocks[t, b] != 0).

Readings where the page leaves a step open:

* ``//`` is floor division (the page's notation is Python's), so a key before
  ``tok_base[t]`` maps to block ``blk_base[t] - 1`` or lower.
* Key tokens range over ``[0, kv_length)``; bounds outside it select nothing
  there.
* ``block_first`` / ``block_last`` describe the block spans for validation by
  the caller; the lookup itself does not read them (the page states the
  relationships as a caller contract that nothing checks).

The allowed set of a query is a set of key tokens, i.e. exactly a route set:
route-set QSA over these sets is the bitmap API's attention.
"""

from __future__ import annotations

import numpy as np


def bitmap_membership(sel_blocks, lo, hi, blk_base, tok_base, kv_length: int, block_size: int = 4) -> np.ndarray:
    """Boolean ``A[t, j]`` = "key token j is allowed for query t" (the lookup, row by row)."""
    sel = np.asarray(sel_blocks)
    T, NB = sel.shape
    lo = np.asarray(lo, dtype=np.int64)
    hi = np.asarray(hi, dtype=np.int64)
    blk_base = np.asarray(blk_base, dtype=np.int64)
    tok_base = np.asarray(tok_base, dtype=np.int64)
    if block_size <= 0:
        raise ValueError("block_size must be positive")
    j = np.arange(kv_length, dtype=np.int64)
    A = np.zeros((T, kv_length), dtype=bool)
    for t in range(T):
        b = blk_base[t] + np.floor_divide(j - tok_base[t], block_size)
        ok = (lo[t] <= j) & (j <= hi[t]) & (b >= 0) & (b < NB)
        bb = np.where(ok, b, 0)
        ok &= sel[t, bb] != 0
        A[t] = ok
    return A


def bitmap_route_rows(sel_blocks, lo, hi, blk_base, tok_base, kv_length: int, block_size: int = 4) -> list:
    """Per query, the ascending allowed key tokens (int64 arrays)."""
    A = bitmap_membership(sel_blocks, lo, hi, blk_base, tok_base, kv_length, block_size)
    return [np.flatnonzero(A[t]) for t in range(A.shape[0])]


def bitmap_routes(sel_blocks, lo, hi, blk_base, tok_base, kv_length: int, width: int, block_size: int = 4):
    """The allowed sets as a ``[T, width]`` int32 route tensor, ascending, -1 padded.

    Returns ``(routes, counts)``; rows with more than ``width`` allowed keys keep
    their ``width`` smallest (``counts`` holds the true sizes).
    """
    rows = bitmap_route_rows(sel_blocks, lo, hi, blk_base, tok_base, kv_length, block_size)
    T = len(rows)
    out = np.full((T, width), -1, dtype=np.int32)
    counts = np.zeros(T, dtype=np.int64)
    for t, r in enumerate(rows):
        counts[t] = r.size
        n = min(r.size, width)
        out[t, :n] = r[:n]
    return out, counts
