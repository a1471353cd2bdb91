"""GPU parity of the QSA selector (tcgen05 scorer, top-k, route expansion).

Defined on the cuDNN-Frontend "Query Sparse Attention (QSA)" page ("Finding
QSA attention and its indexer"); the oracle is ``oracle.qsa_selector``.
Scores: FP32 tensor-core accumulation of BF16 products against the FP64
oracle, max error <= 1e-4 of the row's largest score.  The top-k is an integer
decision taken from floating-point scores, so it is compared bit for bit
against the oracle's top-k applied to the GPU's own FP32 scores (the same
precision on both sides), and the routes against the oracle's expansion.  The
chosen set is also checked against the FP64 oracle scores: it must be a valid
top-k up to the score tolerance (no unchosen candidate beats a chosen one by
more than twice the scores' error bound).
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle.qsa_selector import expand_routes, n_candidates, select, selector_scores, topk_blocks
from token_indexed_sparse_b200 import qsa

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda:0"


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def _check_scores(S_gpu, S_ref, n):
    for t in range(S_ref.shape[0]):
        m = int(n[t])
        if m == 0:
            continue
        a, b = S_gpu[t, :m], S_ref[t, :m]
        assert np.abs(a - b).max() <= 1e-4 * max(np.abs(b).max(), 1e-6), t


def _check_topk_valid(blocks, S_ref, n, k):
    # blocks [T, k] from the GPU against the FP64 scores S_ref: min(k, n_t)
    # distinct candidates, ascending, -1 after them, and a top-k of S_ref up to
    # the tolerance (each side's scores are within 1e-4 of the row maximum)
    for t in range(S_ref.shape[0]):
        m = int(n[t])
        want = min(k, m)
        b = blocks[t]
        chosen = b[:want]
        assert np.all(b[want:] == -1), t
        assert np.all((chosen >= 0) & (chosen < m)) and np.all(np.diff(chosen) > 0), t
        if want == 0 or want == m:
            continue
        row = S_ref[t, :m]
        tol = 2e-4 * max(np.abs(row).max(), 1e-6)
        unchosen = np.setdiff1d(np.arange(m), chosen)
        assert row[chosen].min() >= row[unchosen].max() - tol, t


def _check_topk(S_gpu, n, k, blocks, routes, T, pos=None, tok_base=None):
    ref_b = topk_blocks(S_gpu.astype(np.float64), n, k)
    assert np.array_equal(blocks, ref_b)
    assert np.array_equal(routes, expand_routes(ref_b, T, pos, tok_base))


def test_hand_worked_example_embedded():
    # the 2-head, 2-dim example padded to Hi = 32 heads and Di = 128 dims with
    # zeros: relu(0) = 0, so the scores are unchanged
    fx = json.load(open(os.path.join(HERE, "golden", "selector_example.json")))
    T, NB = fx["T"], len(fx["kbar"])
    qi = np.zeros((T, 32, 128), np.float32)
    qi[:, :2, :2] = np.array(fx["qi"])
    kbar = np.zeros((NB, 128), np.float32)
    kbar[:, :2] = np.array(fx["kbar"])
    S, blocks, routes, status = qsa.select(_bf16(qi).to(DEV), _bf16(kbar).to(DEV), fx["scale"], fx["k"])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    S = S.cpu().numpy()
    for t, v in fx["expected_scores"].items():
        assert np.allclose(S[int(t), :len(v)], v, atol=1e-6), t
    for t, v in fx["expected_blocks"].items():
        assert blocks[int(t)].cpu().tolist() == v, t
    for t, v in fx["expected_routes"].items():
        assert routes[int(t)].cpu().tolist() == v, t


@pytest.mark.parametrize("T,Hi,k,seed", [(300, 64, 16, 1), (1000, 32, 40, 2), (513, 128, 7, 3), (96, 256, 5, 4)])
def test_random_single_sequence(T, Hi, k, seed):
    g = torch.Generator().manual_seed(seed)
    NB = T // 4 + 1
    qi = torch.randn(T, Hi, 128, generator=g).to(torch.bfloat16)
    kbar = torch.randn(NB, 128, generator=g).to(torch.bfloat16)
    scale = 0.125
    S, blocks, routes, status = qsa.select(qi.to(DEV), kbar.to(DEV), scale, k)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    S = S.cpu().numpy()
    n = n_candidates(T, NB)
    S_ref = selector_scores(qi.double().numpy(), kbar.double().numpy(), scale)
    _check_scores(S, S_ref, n)
    _check_topk(S, n, k, blocks.cpu().numpy(), routes.cpu().numpy(), T)
    _check_topk_valid(blocks.cpu().numpy(), S_ref, n, k)


def test_packed_sequences_with_positions():
    # three documents (origins 0, 37, 170), each numbering its own blocks
    g = torch.Generator().manual_seed(7)
    T, Hi, k = 400, 64, 12
    starts = np.array([0, 37, 170])
    doc = np.searchsorted(starts, np.arange(T), side="right") - 1
    tok_base = starts[doc].astype(np.int32)
    nblk = [(37 + 3) // 4, (170 - 37 + 3) // 4, (T - 170 + 3) // 4]
    blk_base = np.array([0, nblk[0], nblk[0] + nblk[1]])[doc].astype(np.int32)
    pos = np.arange(T, dtype=np.int32)
    NB = sum(nblk)
    qi = torch.randn(T, Hi, 128, generator=g).to(torch.bfloat16)
    kbar = torch.randn(NB, 128, generator=g).to(torch.bfloat16)
    d = lambda x: torch.from_numpy(x).to(DEV)  # noqa: E731
    S, blocks, routes, status = qsa.select(qi.to(DEV), kbar.to(DEV), 0.5, k, d(pos), d(blk_base), d(tok_base))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    S = S.cpu().numpy()
    n = n_candidates(T, NB, pos, blk_base, tok_base)
    S_ref = selector_scores(qi.double().numpy(), kbar.double().numpy(), 0.5, pos, blk_base, tok_base)
    _check_scores(S, S_ref, n)
    _check_topk(S, n, k, blocks.cpu().numpy(), routes.cpu().numpy(), T, pos, tok_base)
    _check_topk_valid(blocks.cpu().numpy(), S_ref, n, k)


def test_topk_ties_and_short_rows():
    # scores given directly: many exact ties and rows with fewer candidates than k
    rng = np.random.default_rng(11)
    T, NB, k = 200, 64, 9
    S = rng.integers(0, 4, size=(T, NB)).astype(np.float32)
    blocks, routes = qsa.selector_topk(torch.from_numpy(S).to(DEV), k, NB)
    torch.cuda.synchronize()
    _check_topk(S, n_candidates(T, NB), k, blocks.cpu().numpy(), routes.cpu().numpy(), T)


def test_full_size_sampled_rows():
    # T = 32768 queries, 64 heads x 128 dims, NB = 8192 blocks, k = 127 (+ tail =
    # 128 blocks = 512 route IDs per query, the seq32k attention shape)
    g = torch.Generator().manual_seed(12)
    T, Hi, NB, k = 32768, 64, 8192, 127
    qi = torch.randn(T, Hi, 128, generator=g).to(torch.bfloat16)
    kbar = torch.randn(NB, 128, generator=g).to(torch.bfloat16)
    S, blocks, routes, status = qsa.select(qi.to(DEV), kbar.to(DEV), 1 / 64, k)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(5)
    rows = np.concatenate([[0, 3, 4, 511, 512, 513, T - 1], rng.choice(T, 40, replace=False)])
    kd = kbar.double().numpy()
    Sc, bc, rc = S.cpu().numpy(), blocks.cpu().numpy(), routes.cpu().numpy()
    for t in rows:
        n = min(t // 4, NB)
        if n:
            ref = (1 / 64) * np.maximum(qi[t].double().numpy() @ kd[:n].T, 0).sum(axis=0)
            assert np.abs(Sc[t, :n] - ref).max() <= 1e-4 * np.abs(ref).max(), t
            _check_topk_valid(bc[t:t + 1], ref[None, :], [n], k)
        ref_b = topk_blocks(Sc[t:t + 1].astype(np.float64), [n], k)
        assert np.array_equal(bc[t:t + 1], ref_b), t
        assert np.array_equal(rc[t:t + 1], expand_routes(ref_b, 1, pos=[t])), t


def test_selected_routes_drive_attention():
    # selector routes are valid QSA input: forward runs and every query attends
    # to its causal tail at least
    g = torch.Generator().manual_seed(13)
    T, Hi, k = 256, 32, 8
    qi = torch.randn(T, Hi, 128, generator=g).to(torch.bfloat16).to(DEV)
    kbar = torch.randn(T // 4, 128, generator=g).to(torch.bfloat16).to(DEV)
    _, _, routes, _ = qsa.select(qi, kbar, 0.1, k)
    q = torch.randn(T, 12, 256, generator=g).to(torch.bfloat16).to(DEV)
    kv = torch.randn(T, 1, 256, generator=g).to(torch.bfloat16).to(DEV)
    out, lse = qsa.forward(q, kv, kv, routes, 1 / 16)
    torch.cuda.synchronize()
    assert torch.isfinite(lse).all() and torch.isfinite(out.float()).all()
