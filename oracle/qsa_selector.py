"""Plain CPU restatement of the QSA block selector (scorer, top-k, expansion).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA product path.

Source: cuDNN-Frontend "Query Sparse Attention (QSA)", section "Finding QSA
attention and its indexer": the selector scores each complete compressed block
as ``scale * sum_h relu(qi[t, h] @ kbar[block])`` (compression ratio four,
constant head weights), keeps a ratio-causal top-k, and returns local block
IDs, which need expansion to the attention input format including the
incomplete causal tail and the packed sequence's token origin; and the
"cudnn_qsa" page (``_pack_indices``, ``cudnn_sparse_gqa_attention``): each
four-slot route group is one distinct complete block or the consecutive causal
tail padded with -1, and blocks restart at each packed document origin.

Readings where the pages leave a step open:

* Query t sits at key position ``pos[t]`` of a sequence whose first token is
  ``tok_base[t]`` and whose first compressed block is ``blk_base[t]``; its own
  block is ``o = (pos[t] - tok_base[t]) // 4``.  The candidates are the local
  blocks ``c`` in ``[0, o)`` (complete blocks strictly before the own block);
  local block c is global block ``blk_base[t] + c`` and covers key tokens
  ``tok_base[t] + 4c .. + 3``.
* Candidates must exist: local blocks whose global index ``blk_base + c`` is
  ``>= NB`` are not candidates (the count is ``min(o, NB - blk_base)``).
* Top-k: the k largest scores; equal scores are ordered by the lower local
  block ID.  With fewer than k candidates, all are taken.
* Outputs: the selected local block IDs ascending, -1 padded to k; the routes
  as ``k + 1`` four-slot groups: the selected blocks ascending, then the tail
  (tokens ``tok_base + 4o .. pos[t]``, -1 padded), then -1 groups.

Scores are computed in float64 from the given (BF16-rounded) inputs.
"""

from __future__ import annotations

import numpy as np


def _meta(T, pos, blk_base, tok_base):
    pos = np.arange(T, dtype=np.int64) if pos is None else np.asarray(pos, dtype=np.int64)
    blk_base = np.zeros(T, np.int64) if blk_base is None else np.asarray(blk_base, dtype=np.int64)
    tok_base = np.zeros(T, np.int64) if tok_base is None else np.asarray(tok_base, dtype=np.int64)
    return pos, blk_base, tok_base


def own_blocks(T, pos=None, tok_base=None) -> np.ndarray:
    """Local index of each query's own (tail) block."""
    pos, _, tok_base = _meta(T, pos, None, tok_base)
    return np.maximum((pos - tok_base) // 4, 0)


def n_candidates(T, NB, pos=None, blk_base=None, tok_base=None) -> np.ndarray:
    """Candidates per query: local blocks [0, n) with n = min(own block, NB - blk_base)."""
    pos, blk_base, tok_base = _meta(T, pos, blk_base, tok_base)
    return np.maximum(np.minimum(own_blocks(T, pos, tok_base), NB - blk_base), 0)


def selector_scores(qi, kbar, scale: float, pos=None, blk_base=None, tok_base=None) -> np.ndarray:
    """``S[t, c]`` for the local candidate blocks c < own block (NaN elsewhere).

    ``qi`` is [T, Hi, Di], ``kbar`` is [NB, Di] (global compressed blocks).
    """
    qi = np.asarray(qi, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    T = qi.shape[0]
    pos, blk_base, tok_base = _meta(T, pos, blk_base, tok_base)
    o = n_candidates(T, kbar.shape[0], pos, blk_base, tok_base)
    width = int(max(o.max(initial=0), 0))
    S = np.full((T, width), np.nan)
    for t in range(T):
        n = int(o[t])
        if n <= 0:
            continue
        blocks = kbar[blk_base[t]:blk_base[t] + n]          # [n, Di]
        dots = qi[t] @ blocks.T                             # [Hi, n]
        S[t, :n] = scale * np.maximum(dots, 0.0).sum(axis=0)
    return S


def topk_blocks(S: np.ndarray, n_cand, k: int) -> np.ndarray:
    """Selected local block IDs per row (ascending, -1 padded to k).

    Row t considers ``S[t, :n_cand[t]]``; order: larger score first, then the
    lower block ID.
    """
    T = S.shape[0]
    out = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = int(n_cand[t])
        if n <= 0:
            continue
        c = np.arange(n)
        order = np.lexsort((c, -S[t, :n]))                  # primary: -score, secondary: block ID
        pick = np.sort(order[:k])
        out[t, :pick.size] = pick
    return out


def expand_routes(blocks: np.ndarray, T: int, pos=None, tok_base=None) -> np.ndarray:
    """Token routes [T, 4 (k + 1)] from selected local blocks plus the causal tail."""
    k = blocks.shape[1]
    pos, _, tok_base = _meta(T, pos, None, tok_base)
    out = np.full((T, 4 * (k + 1)), -1, dtype=np.int32)
    for t in range(T):
        sel = blocks[t][blocks[t] >= 0]
        toks = [int(tok_base[t] + 4 * c + i) for c in sel for i in range(4)]
        own = (pos[t] - tok_base[t]) // 4
        tail = list(range(int(tok_base[t] + 4 * own), int(pos[t]) + 1))
        row = toks + tail + [-1] * (4 - len(tail))
        out[t, :len(row)] = row
    return out


def select(qi, kbar, scale: float, k: int, pos=None, blk_base=None, tok_base=None):
    """Scores, selected local blocks and expanded routes: the whole selector."""
    T = np.asarray(qi).shape[0]
    S = selector_scores(qi, kbar, scale, pos, blk_base, tok_base)
    n_cand = n_candidates(T, np.asarray(kbar).shape[0], pos, blk_base, tok_base)
    blocks = topk_blocks(S, n_cand, k)
    return S, blocks, expand_routes(blocks, T, pos, tok_base)
