"""Seeded synthetic QSA workloads (routes and BF16 tensors).

This module only draws inputs; it holds none of the attention arithmetic, so
the CUDA path and the CPU oracle can both be fed from it.

The route structure follows what the documentation pages say about the
ratio-four indexer that produces QSA routes ("cudnn_qsa" page,
``_pack_indices`` and ``cudnn_sparse_gqa_attention``): each four-slot group is
one four-token block, either complete or the query's own causal tail padded
with -1, blocks numbered from each packed document's origin, and -1 rows for
padding queries.  Block choices per configuration:

* ``tiny``   T=256, 12Q/1KV, W=64: min(16, visible) blocks uniform without
  replacement over the visible blocks (the tail may or may not be drawn);
  the last 8 rows all -1.
* ``seq4k``  T=4096, 12Q/1KV, W=256: 64 distinct blocks, the own (tail) block
  always, the rest uniform over the earlier visible blocks.
* ``thd16k`` T=16384 packed as 8 documents (7 distinct sorted cut points
  uniform in [1, T-1], redrawn while a document is shorter than 4 tokens),
  W=512: 128 blocks within the query's document, own block always; a seeded
  3% of rows all -1.
* ``seq32k`` T=32768, 24Q/2KV (routes shared by both groups), W=564: 128
  distinct blocks, 64 from the 512 most recent blocks (own block always) and
  64 uniform over the older visible blocks; where a pool is short the other
  pool makes up the count.  Then ceil(10%) of each row's valid IDs are
  appended again as duplicates and the row is shuffled.
* ``cp128k`` 8192 local queries at global positions 122880..131071 against
  131072 K/V rows, 12Q/1KV, W=2048: 512 distinct blocks, own block always,
  the others without replacement with weight d^-1.1 in the block distance
  d >= 1; a seeded 5% of rows all -1.

Seeds are 1001 to 1005, in the order above.  Routes come from numpy's PCG64; q, k, v and
grad_out are N(0, 1) float32 draws from a seeded torch CPU generator, rounded
once to BF16 (the BF16 values are what both sides consume).
"""

from __future__ import annotations

import dataclasses
import functools
import math

import numpy as np

HEAD_DIM = 256


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    T_kv: int
    H: int
    G: int
    W: int
    blocks: int            # target distinct blocks per query
    policy: str            # "uniform", "own_uniform", "near_far", "zipf"
    q_offset: int = 0      # global position of the first query row
    n_docs: int = 1
    pad_frac: float = 0.0  # fraction of rows that are all -1
    pad_tail: int = 0      # number of trailing rows that are all -1
    dup_frac: float = 0.0
    scale: float = 1.0 / 16.0
    seed: int = 0

    @property
    def D(self) -> int:
        return HEAD_DIM

    def scaled(self, T: int, T_kv: int | None = None, blocks: int | None = None,
               W: int | None = None) -> "Workload":
        """The same recipe at a smaller size (used for exhaustive parity runs)."""
        if T_kv is None:
            T_kv = T if self.q_offset == 0 else T * (self.T_kv // self.T)
        return dataclasses.replace(
            self, name=f"{self.name}@{T}", T=T, T_kv=T_kv,
            q_offset=(T_kv - T) if self.q_offset else 0,
            blocks=self.blocks if blocks is None else blocks,
            W=self.W if W is None else W,
            pad_tail=min(self.pad_tail, T // 4))


WORKLOADS = {
    "tiny": Workload("tiny", 256, 256, 12, 1, 64, 16, "uniform", pad_tail=8, seed=1001),
    "seq4k": Workload("seq4k", 4096, 4096, 12, 1, 256, 64, "own_uniform", seed=1002),
    "thd16k": Workload("thd16k", 16384, 16384, 12, 1, 512, 128, "own_uniform", n_docs=8,
                         pad_frac=0.03, seed=1003),
    "seq32k": Workload("seq32k", 32768, 32768, 24, 2, 564, 128, "near_far", dup_frac=0.10,
                         seed=1004),
    "cp128k": Workload("cp128k", 8192, 131072, 12, 1, 2048, 512, "zipf", q_offset=122880,
                         pad_frac=0.05, seed=1005),
}


def _doc_starts(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    if wl.n_docs <= 1:
        return np.array([0], dtype=np.int64)
    while True:
        cuts = np.sort(rng.choice(np.arange(1, wl.T_kv), wl.n_docs - 1, replace=False))
        starts = np.concatenate([[0], cuts])
        lengths = np.diff(np.concatenate([starts, [wl.T_kv]]))
        if lengths.min() >= 4:
            return starts.astype(np.int64)


def _zipf_pick(rng, own: int, n: int, s: float = 1.1) -> np.ndarray:
    """n distinct blocks from [0, own) with weight (own - b)^-s (Gumbel top-k)."""
    if n <= 0 or own <= 0:
        return np.zeros(0, dtype=np.int64)
    if n >= own:
        return np.arange(own, dtype=np.int64)
    d = own - np.arange(own, dtype=np.float64)
    keys = -s * np.log(d) - np.log(-np.log(rng.random(own)))
    return np.argpartition(-keys, n - 1)[:n].astype(np.int64)


def _pick_blocks(wl: Workload, rng, own: int) -> np.ndarray:
    """Doc-local block indices for a query whose own (tail) block is ``own``."""
    visible = own + 1
    if wl.policy == "uniform":
        return rng.choice(visible, min(wl.blocks, visible), replace=False).astype(np.int64)
    if wl.policy == "own_uniform":
        n_other = min(wl.blocks, visible) - 1
        others = rng.choice(own, n_other, replace=False) if n_other > 0 else np.zeros(0, np.int64)
        return np.concatenate([[own], others]).astype(np.int64)
    if wl.policy == "near_far":
        near_lo = max(0, own - 511)
        n_near_avail = own - near_lo          # near blocks besides the own block
        n_far_avail = near_lo                 # blocks older than the window
        half = wl.blocks // 2
        n_far = min(half, n_far_avail)
        n_near = min(wl.blocks - n_far - 1, n_near_avail)
        n_far = min(wl.blocks - 1 - n_near, n_far_avail)
        near = near_lo + rng.choice(n_near_avail, n_near, replace=False) if n_near > 0 else np.zeros(0, np.int64)
        far = rng.choice(n_far_avail, n_far, replace=False) if n_far > 0 else np.zeros(0, np.int64)
        return np.concatenate([[own], near, far]).astype(np.int64)
    if wl.policy == "zipf":
        n_other = min(wl.blocks, visible) - 1
        return np.concatenate([[own], _zipf_pick(rng, own, n_other)]).astype(np.int64)
    raise ValueError(wl.policy)


@functools.lru_cache(maxsize=16)
def make_routes(wl: Workload) -> np.ndarray:
    """Route IDs ``[T, W]`` int32 for a workload (cached; treat as read-only)."""
    rng = np.random.default_rng(wl.seed)
    starts = _doc_starts(wl, rng)
    routes = np.full((wl.T, wl.W), -1, dtype=np.int32)
    slot = np.arange(4, dtype=np.int64)
    for t in range(wl.T):
        pos = wl.q_offset + t                       # global position of the query
        doc = starts[np.searchsorted(starts, pos, side="right") - 1]
        own = (pos - doc) // 4
        blocks = rng.permutation(_pick_blocks(wl, rng, int(own)))
        ids = doc + 4 * blocks[:, None] + slot[None, :]
        ids = np.where(ids <= pos, ids, -1).reshape(-1)
        if wl.dup_frac > 0:
            valid = ids[ids >= 0]
            n_dup = min(int(math.ceil(wl.dup_frac * len(valid))), wl.W - len(ids))
            if n_dup > 0:
                ids = np.concatenate([ids, rng.choice(valid, n_dup, replace=True)])
            ids = rng.permutation(ids)
        n = min(len(ids), wl.W)
        routes[t, :n] = ids[:n]
    if wl.pad_frac > 0:
        n_pad = int(math.floor(wl.pad_frac * wl.T))
        routes[rng.choice(wl.T, n_pad, replace=False)] = -1
    if wl.pad_tail > 0:
        routes[wl.T - wl.pad_tail:] = -1
    routes.setflags(write=False)
    return routes


def make_tensors(wl: Workload, with_grad: bool = True):
    """q ``[T,H,256]``, k, v ``[T_kv,G,256]`` (and grad_out) as BF16 CPU tensors."""
    import torch

    g = torch.Generator().manual_seed(wl.seed)

    def draw(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)

    q = draw(wl.T, wl.H, HEAD_DIM)
    k = draw(wl.T_kv, wl.G, HEAD_DIM)
    v = draw(wl.T_kv, wl.G, HEAD_DIM)
    do = draw(wl.T, wl.H, HEAD_DIM) if with_grad else None
    return q, k, v, do


def pair_count(routes: np.ndarray, T_kv: int) -> int:
    """N = sum over rows of |R_t| (unique valid route IDs)."""
    r = np.asarray(routes).astype(np.int64)
    valid = (r >= 0) & (r < T_kv)
    key = np.where(valid, r, -1)
    key = np.sort(key, axis=1)
    distinct = (key[:, 1:] != key[:, :-1]) & (key[:, 1:] >= 0)
    return int(distinct.sum() + (key[:, 0] >= 0).sum())


def make_bitmap_case(T: int, n_docs: int, blocks_per_row: int, seed: int, block_size: int = 4,
                     perturb_frac: float = 0.05) -> dict:
    """A seeded packed-sequence input in the bitmap selection format.

    ``T`` tokens are cut into ``n_docs`` documents at sorted distinct cut points
    (document origins need not be multiples of ``block_size``).  Each document
    numbers its own blocks from its origin; the last block of a document may be
    short.  Query t gets ``lo`` = its document's origin, ``hi`` = t, the
    document's ``blk_base`` / ``tok_base``, and ``blocks_per_row`` selected
    blocks drawn uniformly from all NB global blocks (so some fall outside its
    bounds or document).  A seeded ``perturb_frac`` of rows gets bounds that
    stray outside the document or are empty (lo > hi).  Returns numpy arrays
    ``sel_blocks [T, NB] uint8, lo, hi, blk_base, tok_base [T] int32,
    block_first, block_last [NB] int32`` and ``T_kv = T``.
    """
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.choice(np.arange(1, T), size=n_docs - 1, replace=False)) if n_docs > 1 else np.array([], int)
    starts = np.concatenate([[0], cuts]).astype(np.int64)
    ends = np.concatenate([cuts, [T]]).astype(np.int64)
    block_first, block_last, doc_blk = [], [], []
    for s, e in zip(starts, ends):
        doc_blk.append(len(block_first))
        for b0 in range(s, e, block_size):
            block_first.append(b0)
            block_last.append(min(b0 + block_size, e) - 1)
    NB = len(block_first)
    doc_of = np.searchsorted(ends, np.arange(T), side="right")
    lo = starts[doc_of].astype(np.int32)
    hi = np.arange(T, dtype=np.int32)
    blk_base = np.array(doc_blk, dtype=np.int32)[doc_of]
    tok_base = starts[doc_of].astype(np.int32)
    sel = np.zeros((T, NB), dtype=np.uint8)
    k = min(blocks_per_row, NB)
    for t in range(T):
        sel[t, rng.choice(NB, size=k, replace=False)] = 1
    n_pert = int(perturb_frac * T)
    rows = rng.choice(T, size=n_pert, replace=False)
    for i, t in enumerate(rows):
        if i % 3 == 0:
            lo[t] = max(0, int(lo[t]) - int(rng.integers(1, 9)))   # reaches into the previous document
        elif i % 3 == 1:
            lo[t] = hi[t] + 1                                        # empty bounds
        else:
            hi[t] = min(T - 1, int(hi[t]) + int(rng.integers(1, 9)))  # beyond the query
    return {"sel_blocks": sel, "lo": lo, "hi": hi, "blk_base": blk_base, "tok_base": tok_base,
            "block_first": np.array(block_first, np.int32), "block_last": np.array(block_last, np.int32),
            "T_kv": T, "NB": NB}
