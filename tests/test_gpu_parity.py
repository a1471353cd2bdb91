"""GPU parity: the CUDA path through the C ABI against the FP64 CPU oracle.

Tolerances (from the workload statement): out/dq/dk/dv max |gpu - oracle| /
max |oracle| <= 1e-2 per tensor; LSE absolute error <= 1e-3 on non-empty rows
and exactly -inf on empty rows.  Index work (route preprocessing) is bit-exact.
"""

import numpy as np
import pytest
import torch

import oracle
from token_indexed_sparse_b200 import qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2
LSE_TOL = 1e-3
DEV = torch.device("cuda:0")


def f64(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    # max |got - ref| / max |ref|; a reference that is zero to within 1e-3 everywhere
    # (e.g. dQ of single-key rows, exactly 0 in exact arithmetic) is compared with an
    # absolute floor of 1e-3 instead of dividing by ~0.
    return np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-3)


def to_dev(routes, *tensors):
    r = torch.from_numpy(np.array(routes, dtype=np.int32)).to(DEV)
    return (r, *[t.to(DEV) for t in tensors])


def status_word(ws):
    # the first int32 of a workspace: 0 unless a kernel gave up on a bounded wait
    return int(ws[:4].view(torch.int32).item())


def run_gpu(q, k, v, do, routes, scale):
    r, qd, kd, vd, dod = to_dev(routes, q, k, v, do)
    T, H = qd.shape[0], qd.shape[1]
    ws = torch.empty(qsa.backward_workspace_size(T, kd.shape[0], H, kd.shape[1], r.shape[1]),
                     dtype=torch.uint8, device=DEV)
    out, lse = qsa.forward(qd, kd, vd, r, scale)
    dq, dk, dv = qsa.backward(dod, qd, kd, vd, out, lse, r, scale, workspace=ws)
    torch.cuda.synchronize()
    assert status_word(ws) == 0
    return out, lse, dq, dk, dv


def check_lse(got, ref):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.all(got[~fin] == -np.inf)
    if fin.any():
        assert np.abs(got[fin] - ref[fin]).max() <= LSE_TOL


def check_all(res, ref):
    out, lse, dq, dk, dv = res
    r_out, r_lse, r_dq, r_dk, r_dv = ref
    check_lse(lse.cpu().numpy().astype(np.float64), r_lse)
    for name, g, r in (("out", out, r_out), ("dq", dq, r_dq), ("dk", dk, r_dk), ("dv", dv, r_dv)):
        e = rel_err(f64(g), r)
        assert e <= REL_TOL, f"{name}: relative max error {e:.3e}"


def inputs(wl):
    routes = W.make_routes(wl)
    q, k, v, do = W.make_tensors(wl)
    return routes, q, k, v, do


# ---------------------------------------------------------------------------
# exhaustive parity on every workload recipe at sizes the dense oracle finishes
# ---------------------------------------------------------------------------

SMALL = {"tiny": None, "seq4k": 512, "thd16k": 1024, "seq32k": 768, "cp128k": 256}


@pytest.mark.parametrize("name", list(SMALL))
def test_parity_dense_oracle(name):
    wl = W.WORKLOADS[name] if SMALL[name] is None else W.WORKLOADS[name].scaled(SMALL[name])
    routes, q, k, v, do = inputs(wl)
    res = run_gpu(q, k, v, do, routes, wl.scale)
    ref_out, ref_lse = oracle.forward_dense(f64(q), f64(k), f64(v), routes, wl.scale)
    ref_g = oracle.backward_dense(f64(do), f64(q), f64(k), f64(v), routes, wl.scale)
    check_all(res, (ref_out, ref_lse, *ref_g))
    # padding rows: exact zeros; untouched keys: exact zeros
    out, lse, dq, dk, dv = res
    empty = ~oracle.routes_to_membership(routes, wl.T_kv).any(axis=1)
    assert torch.all(out[torch.from_numpy(empty)] == 0) and torch.all(dq[torch.from_numpy(empty)] == 0)
    touched = oracle.routes_to_membership(routes, wl.T_kv).any(axis=0)
    assert torch.all(dk[torch.from_numpy(~touched)] == 0) and torch.all(dv[torch.from_numpy(~touched)] == 0)


# ---------------------------------------------------------------------------
# full workload sizes: sampled rows and keys computed one by one by the oracle
# ---------------------------------------------------------------------------

def phase_spanning_tiles(routes, T_kv, C, n=2):
    """Two 128-key tiles whose query lists reach into at least two dK/dV query
    phases of C rows (so their dK/dV sum ordered FP32 partials across phases),
    the ones with the median number of (query, tile) entries among those
    (when T <= C there is one phase: the median tiles with entries)."""
    r = np.asarray(routes).astype(np.int64)
    t = np.repeat(np.arange(r.shape[0], dtype=np.int64), r.shape[1])
    key = r.ravel()
    ok = (key >= 0) & (key < T_kv)
    pair = np.unique(t[ok] * ((T_kv + 127) // 128) + key[ok] // 128)   # distinct (query, tile)
    tq, tl = pair // ((T_kv + 127) // 128), pair % ((T_kv + 127) // 128)
    n_ent = np.bincount(tl, minlength=(T_kv + 127) // 128)
    phases = np.unique(tl * (1 << 20) + tq // C)
    n_ph = np.bincount(phases >> 20, minlength=(T_kv + 127) // 128)
    multi = np.nonzero(n_ph >= 2)[0]
    if len(multi) < n:                      # a single phase (T <= C): any tiles with entries
        multi = np.nonzero(n_ent > 0)[0]
    order = multi[np.argsort(n_ent[multi], kind="stable")]
    mid = len(order) // 2
    return order[mid : mid + n]


def dkdv_phase_rows(T, H):
    # the library's dK/dV query-phase length: 48 MiB of one tensor's Q rows,
    # at least 4096 rows, a multiple of 256 (at most 64 phases)
    c = (48 << 20) // (H * 1024)
    c = 4096 if c < 4096 else (c // 256) * 256
    if (T + c - 1) // c > 64:
        c = (((T + 63) // 64) + 255) // 256 * 256
    return c


@pytest.mark.parametrize("name", ["seq4k", "thd16k", "seq32k", "cp128k"])
def test_parity_full_size_sampled(name):
    wl = W.WORKLOADS[name]
    routes, q, k, v, do = inputs(wl)
    out, lse, dq, dk, dv = run_gpu(q, k, v, do, routes, wl.scale)
    rng = np.random.default_rng(wl.seed - 1000)
    counts = oracle.route_rows_csr(routes, wl.T_kv)[0]
    rows = np.unique(np.concatenate([rng.choice(wl.T, 509, replace=False),
                                     [int(np.argmax(counts)), wl.T - 1, 0]]))
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    r_out, r_lse = oracle.forward_rows(qf, kf, vf, routes, wl.scale, rows)
    r_dq, _, _ = oracle.backward_rows(dof, qf, kf, vf, routes, wl.scale, rows)
    check_lse(lse[rows].cpu().numpy().astype(np.float64), r_lse)
    assert rel_err(f64(out[rows]), r_out) <= REL_TOL
    assert rel_err(f64(dq[rows]), r_dq) <= REL_TOL
    # keys: random, the most recent (hot) ones, one past every route, and every
    # key of two whole 128-key tiles whose dK/dV sums run over several query
    # phases (ordered FP32 partials between phases)
    tiles = phase_spanning_tiles(routes, wl.T_kv, dkdv_phase_rows(wl.T, wl.H))
    keys = np.unique(np.concatenate([rng.choice(wl.T_kv, 10, replace=False),
                                     [wl.T_kv - 1, wl.T_kv - 5]] +
                                    [np.arange(tl * 128, min(wl.T_kv, tl * 128 + 128)) for tl in tiles]))
    r_dk, r_dv = oracle.backward_keys(dof, qf, kf, vf, routes, wl.scale, keys)
    assert rel_err(f64(dk[keys]), r_dk) <= REL_TOL
    assert rel_err(f64(dv[keys]), r_dv) <= REL_TOL
    # properties over the whole output
    empty = torch.from_numpy(counts == 0)
    assert torch.all(out[empty] == 0) and torch.all(dq[empty] == 0)
    assert torch.all(torch.isneginf(lse[empty])) and torch.all(torch.isfinite(lse[~empty]))
    assert torch.isfinite(out).all() and torch.isfinite(dq).all()
    assert torch.isfinite(dk).all() and torch.isfinite(dv).all()


# ---------------------------------------------------------------------------
# route preprocessing: bit-exact
# ---------------------------------------------------------------------------

def _check_plan(routes, T_kv):
    r = torch.from_numpy(np.array(routes, dtype=np.int32)).to(DEV)
    row_cnt, row_cols, quad_ptr, quad_ent = (x.cpu().numpy() for x in qsa.route_plan(r, T_kv))
    cnt, cols = oracle.route_rows_csr(routes, T_kv)
    np.testing.assert_array_equal(row_cnt, cnt)
    for t in range(len(cnt)):
        np.testing.assert_array_equal(row_cols[t, :cnt[t]], cols[t, :cnt[t]])
    ptr, qry, msk = oracle.key_quad_lists(routes, T_kv)
    np.testing.assert_array_equal(quad_ptr, ptr)
    ent = quad_ent[: ptr[-1]]
    np.testing.assert_array_equal(ent >> 32, qry)
    np.testing.assert_array_equal(ent & 15, msk)
    # i0: position in R_t of the quad's first routed key
    quad_of = np.repeat(np.arange(len(ptr) - 1), np.diff(ptr))
    first_key = 4 * quad_of + np.array([(int(m) & -int(m)).bit_length() - 1 for m in msk], dtype=np.int64)
    i0 = np.array([np.searchsorted(cols[t, :cnt[t]], j) for t, j in zip(qry, first_key)])
    np.testing.assert_array_equal((ent >> 4) & 0x0FFFFFFF, i0)


@pytest.mark.parametrize("name,T", list(SMALL.items()))
def test_route_plan_bitexact(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].scaled(T)
    _check_plan(W.make_routes(wl), wl.T_kv)


def test_route_plan_edge_rows():
    rng = np.random.default_rng(5)
    T, T_kv = 300, 41                                   # ragged last quad (key 40 alone)
    routes = rng.integers(-50, T_kv + 50, size=(T, 37)).astype(np.int32)
    routes[3] = -1
    routes[4] = 40
    routes[5, :] = [2**31 - 1, -2**31] * 18 + [7]
    routes[6] = np.arange(37) % 4                       # duplicates of one quad
    _check_plan(routes, T_kv)


@pytest.mark.parametrize("n_sel", [2, 33, 64, 65, 300, 512, 513, 544, 545, 576, 577, 640, 641, 700, 768, 769,
                                   1024, 1025, 2048])
def test_route_rows_every_kernel_width(n_sel):
    # the route-row kernels change with n_sel (register networks of 64 .. 1024
    # slots, 512 + 32 .. 512 + 256 split sorts merged in shared memory, and the
    # CTA sort above 1024): rows with duplicates, invalid IDs, empty rows and
    # rows that fill every slot with distinct keys
    rng = np.random.default_rng(n_sel)
    T, T_kv = 96, 3000
    routes = rng.integers(-40, T_kv + 40, size=(T, n_sel)).astype(np.int32)
    routes[0] = -1
    routes[1] = rng.permutation(T_kv)[:n_sel] if n_sel <= T_kv else routes[1]
    routes[2] = 7
    routes[3, : n_sel // 2] = routes[3, n_sel - n_sel // 2:] if n_sel > 1 else routes[3, :0]
    routes[4] = np.sort(routes[4])[::-1]
    _check_plan(routes, T_kv)


def test_route_plan_long_quad_list():
    # 5000 queries share one quad: its list is longer than the in-shared-memory sort
    T, T_kv = 5000, 16
    routes = np.tile(np.array([[3, 1, 2, 0, -1]], dtype=np.int32), (T, 1))
    routes[::7, 0] = 9
    _check_plan(routes, T_kv)


def _check_tile_plan(routes, T_kv):
    r = torch.from_numpy(np.array(routes, dtype=np.int32)).to(DEV)
    row_cnt, row_cols, tile_ptr, tile_ent = (x.cpu().numpy() for x in qsa.tile_plan(r, T_kv))
    cnt, cols = oracle.route_rows_csr(routes, T_kv)
    np.testing.assert_array_equal(row_cnt, cnt)
    ptr, qry, i0, n = oracle.key_tile_lists(routes, T_kv)
    np.testing.assert_array_equal(tile_ptr, ptr)
    ent = tile_ent[: ptr[-1]]
    np.testing.assert_array_equal(ent >> 32, qry)
    np.testing.assert_array_equal((ent >> 8) & 0x3FFF, i0)
    np.testing.assert_array_equal((ent & 0x7F) + 1, n)


@pytest.mark.parametrize("name,T", list(SMALL.items()))
def test_tile_plan_bitexact(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].scaled(T)
    _check_tile_plan(W.make_routes(wl), wl.T_kv)


def test_tile_plan_edge_rows():
    rng = np.random.default_rng(6)
    T, T_kv = 300, 397                                  # ragged last tile (keys 384..396)
    routes = rng.integers(-50, T_kv + 50, size=(T, 150)).astype(np.int32)
    routes[3] = -1
    routes[4] = 396
    routes[5, :128] = np.arange(128, 256)               # one full tile: n = 128
    routes[5, 128:] = -1
    routes[6] = np.arange(150) % 5                      # duplicates inside one tile
    _check_tile_plan(routes, T_kv)


def test_tile_plan_long_list():
    # 20000 queries meet tile 0: its list is longer than the in-shared-memory sort
    T, T_kv = 20000, 300
    routes = np.tile(np.array([[3, 1, 200, 0, -1]], dtype=np.int32), (T, 1))
    routes[::7, 0] = 299
    _check_tile_plan(routes, T_kv)


def test_tile_plan_many_tiles():
    # more tiles than the shared-memory histograms hold (global-atomic path)
    rng = np.random.default_rng(8)
    T, T_kv = 64, 128 * 9000
    routes = rng.integers(0, T_kv, size=(T, 40)).astype(np.int32)
    _check_tile_plan(routes, T_kv)


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def _rand_inputs(T, T_kv, G, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)  # noqa: E731
    return mk(T, 12 * G, 256), mk(T_kv, G, 256), mk(T_kv, G, 256), mk(T, 12 * G, 256)


def _dense_ref(q, k, v, do, routes, scale):
    out, lse = oracle.forward_dense(f64(q), f64(k), f64(v), routes, scale)
    return (out, lse, *oracle.backward_dense(f64(do), f64(q), f64(k), f64(v), routes, scale))


@pytest.mark.parametrize("case", ["single", "all_empty", "ragged_kv", "noncausal", "dups_invalid",
                                  "wide_row", "max_n_sel", "one_hot_key", "g2_shared"])
def test_edge_cases(case):
    rng = np.random.default_rng(hash(case) % 2**32)
    scale = 1.0 / 16
    G = 1
    if case == "single":
        T, T_kv = 1, 1
        routes = np.array([[0]], np.int32)
    elif case == "all_empty":
        T, T_kv = 40, 40
        routes = np.full((T, 8), -1, np.int32)
    elif case == "ragged_kv":
        T, T_kv = 70, 5
        routes = rng.integers(-2, 7, size=(T, 6)).astype(np.int32)
    elif case == "noncausal":
        T, T_kv = 64, 64
        routes = rng.integers(0, T_kv, size=(T, 40)).astype(np.int32)   # future keys allowed
    elif case == "dups_invalid":
        T, T_kv = 50, 33
        routes = rng.integers(0, T_kv, size=(T, 5)).astype(np.int32)
        routes = np.concatenate([routes, routes, np.full((T, 3), -5, np.int32),
                                 np.tile(np.array([[33, 40, 2**31 - 1, -2**31]], np.int32), (T, 1))], 1)
    elif case == "wide_row":
        T, T_kv = 24, 700
        routes = rng.integers(-100, T_kv, size=(T, 3000)).astype(np.int32)   # ~all keys, many dups
    elif case == "max_n_sel":
        T, T_kv = 8, 300
        routes = np.full((T, 16384), -1, np.int32)
        routes[:, ::97] = rng.integers(0, T_kv, size=(T, len(range(0, 16384, 97))))
    elif case == "one_hot_key":
        T, T_kv = 600, 12
        routes = np.full((T, 4), -1, np.int32)
        routes[:, 0] = 5
        routes[::3, 1] = 6
    elif case == "g2_shared":
        T, T_kv, G = 90, 90, 2
        routes = rng.integers(-1, T_kv, size=(T, 33)).astype(np.int32)
    q, k, v, do = _rand_inputs(T, T_kv, G, 7)
    res = run_gpu(q, k, v, do, routes, scale)
    check_all(res, _dense_ref(q, k, v, do, routes, scale))
    if case == "single":
        out, lse, dq, dk, dv = res
        assert torch.equal(out.cpu()[0], v[0].expand(12, 256))          # P = 1 exactly
        assert dq.abs().max() < 1e-4 and dk.abs().max() < 1e-4            # dS = 0 up to rounding


# ---------------------------------------------------------------------------
# determinism, non-finite isolation, error statuses
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["thd16k", "seq32k"])  # 1 KV group, 4 dK/dV phases; 2 groups, 8 phases
def test_backward_is_bitwise_deterministic(name):
    wl = W.WORKLOADS[name]
    routes, q, k, v, do = inputs(wl)
    r, qd, kd, vd, dod = to_dev(routes, q, k, v, do)
    out, lse = qsa.forward(qd, kd, vd, r, wl.scale)
    ws = torch.empty(qsa.backward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, routes.shape[1]),
                     dtype=torch.uint8, device=DEV)
    first = qsa.backward(dod, qd, kd, vd, out, lse, r, wl.scale)
    for _ in range(2):
        again = qsa.backward(dod, qd, kd, vd, out, lse, r, wl.scale, workspace=ws)
        torch.cuda.synchronize()
        assert status_word(ws) == 0
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    out2, lse2 = qsa.forward(qd, kd, vd, r, wl.scale)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_unselected_nonfinite_kv_never_read():
    wl = W.WORKLOADS["seq4k"].scaled(512)
    routes, q, k, v, do = inputs(wl)
    rng = np.random.default_rng(2)
    unused = np.sort(rng.choice(wl.T_kv, 64, replace=False))
    routes = np.where(np.isin(routes, unused), -1, routes).astype(np.int32)
    used = np.unique(routes[routes >= 0])
    assert len(np.intersect1d(used, unused)) == 0
    k2, v2 = k.clone(), v.clone()
    k2[torch.from_numpy(unused)] = float("nan")
    v2[torch.from_numpy(unused[::2])] = float("inf")
    a = run_gpu(q, k, v, do, routes, wl.scale)
    b = run_gpu(q, k2, v2, do, routes, wl.scale)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    ut = torch.from_numpy(used).to(DEV)
    assert torch.equal(a[3][ut], b[3][ut]) and torch.equal(a[4][ut], b[4][ut])
    un = torch.from_numpy(unused).to(DEV)
    assert torch.all(b[3][un] == 0) and torch.all(b[4][un] == 0)


def test_error_statuses_launch_nothing():
    T, T_kv = 32, 32
    q, k, v, do = (x.to(DEV) for x in _rand_inputs(T, T_kv, 1, 3))
    routes = torch.zeros(T, 4, dtype=torch.int32, device=DEV)
    out = torch.full_like(q, 7.0)
    lse = torch.full((T, 12), 7.0, device=DEV)
    lib = qsa.library()
    ws = torch.empty(lib.qsa_forward_workspace_size(T, T_kv, 12, 1, 4), dtype=torch.uint8, device=DEV)
    P = lambda t, off=0: __import__("ctypes").c_void_p(t.data_ptr() + off)  # noqa: E731
    S = __import__("ctypes").c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.qsa_forward(P(q), P(k), P(v), P(routes), T, T_kv, 12, 1, 4, 0.0625, P(out), P(lse), P(ws),
                         ws.numel() - 1, S)
    assert st == 4
    st = lib.qsa_forward(P(q, 2), P(k), P(v), P(routes), T, T_kv, 12, 1, 4, 0.0625, P(out), P(lse), P(ws),
                         ws.numel(), S)
    assert st == 3
    st = lib.qsa_forward(P(q), P(k), P(v), P(routes), T, T_kv, 24, 1, 4, 0.0625, P(out), P(lse), P(ws),
                         ws.numel(), S)
    assert st == 2
    torch.cuda.synchronize()
    assert torch.all(out == 7.0) and torch.all(lse == 7.0)
    with pytest.raises(qsa.QSAError):
        qsa.forward(q, k, v, routes, scale=float("nan"))


# ---------------------------------------------------------------------------
# query-union lists (the forward's key lists): bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,T", [("tiny", None), ("seq4k", 512), ("thd16k", 1024), ("seq32k", 768),
                                    ("cp128k", 256)])
def test_union_plan_bitexact(name, T):
    wl = W.WORKLOADS[name] if T is None else W.WORKLOADS[name].scaled(T)
    routes = W.make_routes(wl)
    if name == "tiny":
        routes = np.array(routes)
        routes[10] = routes[11]                    # two rows of one group with the same set
        routes[13, :5] = [7, 7, -1, wl.T_kv, 200]  # duplicates and invalid IDs
    r = torch.from_numpy(np.array(routes, dtype=np.int32)).to(DEV)
    group, ucnt, ukey, uown = qsa.union_plan(r, wl.T_kv)
    torch.cuda.synchronize()
    cnt, keys, owners = oracle.query_union_lists(routes, wl.T_kv, group)
    np.testing.assert_array_equal(ucnt.cpu().numpy(), cnt)
    ukey, uown = ukey.cpu().numpy(), uown.cpu().numpy()
    for i in range(len(cnt)):
        np.testing.assert_array_equal(ukey[i, :cnt[i]], keys[i])
        np.testing.assert_array_equal(uown[i, :cnt[i]], owners[i])


def test_union_plan_long_rows_fall_back_to_single_rows():
    # rows of more than 4096 slots are not merged (groups of one row)
    rng = np.random.default_rng(5)
    T, T_kv, n_sel = 20, 50000, 5000
    routes = rng.integers(-10, T_kv, size=(T, n_sel)).astype(np.int32)
    r = torch.from_numpy(routes).to(DEV)
    group, ucnt, ukey, uown = qsa.union_plan(r, T_kv)
    torch.cuda.synchronize()
    assert group == 1
    cnt, keys, owners = oracle.query_union_lists(routes, T_kv, 1)
    np.testing.assert_array_equal(ucnt.cpu().numpy(), cnt)
    for i in range(T):
        np.testing.assert_array_equal(ukey[i, :cnt[i]].cpu().numpy(), keys[i])
        assert np.all(uown[i, :cnt[i]].cpu().numpy() == 1)
