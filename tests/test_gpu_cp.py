"""GPU checks of the FP32 dK/dV backward and of the context-parallel path.

With one GPU the process group has one rank: the all-gather and the
reduce-scatter are identities, so the CP path must reproduce the plain calls
bit for bit.  The FP32 dK/dV backward ("Query Sparse Attention (QSA)" page,
"Selection and components": FP32 accumulation) must round to exactly the BF16
backward's dK/dV and match the oracle.  The collective plumbing over several
ranks is covered on CPU processes (tests/test_cp.py).
"""

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import backward_dense
from token_indexed_sparse_b200 import cp, qsa
from token_indexed_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(name, T):
    wl = W.WORKLOADS[name].scaled(T)
    routes = torch.from_numpy(np.array(W.make_routes(wl))).to(DEV)
    q, k, v, do = (x.to(DEV) for x in W.make_tensors(wl))
    return wl, routes, q, k, v, do


@pytest.mark.parametrize("name,T", [("thd16k", 1024), ("cp128k", 256)])
def test_fp32_kv_backward(name, T):
    wl, routes, q, k, v, do = _inputs(name, T)
    out, lse = qsa.forward(q, k, v, routes, wl.scale)
    dq, dk, dv = qsa.backward(do, q, k, v, out, lse, routes, wl.scale)
    dq32, dk32, dv32 = qsa.backward(do, q, k, v, out, lse, routes, wl.scale, kv_fp32=True)
    torch.cuda.synchronize()
    assert dk32.dtype == torch.float32 and dv32.dtype == torch.float32
    assert torch.equal(dq32, dq)
    assert torch.equal(dk32.to(torch.bfloat16), dk) and torch.equal(dv32.to(torch.bfloat16), dv)
    r = routes.cpu().numpy()
    _, o_dk, o_dv = backward_dense(do.double().cpu().numpy(), q.double().cpu().numpy(), k.double().cpu().numpy(),
                                   v.double().cpu().numpy(), r, wl.scale)
    for a, b in ((dk32, o_dk), (dv32, o_dv)):
        a = a.double().cpu().numpy()
        assert np.abs(a - b).max() / max(np.abs(b).max(), 1e-3) <= 1e-2


def test_cp_single_rank_reproduces_plain_calls():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device(DEV))
    try:
        wl, routes, q, k, v, do = _inputs("cp128k", 512)
        out, lse = qsa.forward(q, k, v, routes, wl.scale)
        dq, dk, dv = qsa.backward(do, q, k, v, out, lse, routes, wl.scale)
        c_out, c_lse = cp.cp_forward(q, k, v, routes, wl.scale)
        c_dq, c_dk, c_dv = cp.cp_backward(do, q, k, v, c_out, c_lse, routes, wl.scale)
        torch.cuda.synchronize()
        assert torch.equal(c_out, out) and torch.equal(c_lse, lse)
        assert torch.equal(c_dq, dq) and torch.equal(c_dk, dk) and torch.equal(c_dv, dv)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kv_fp32", [False, True])
def test_kv_ready_event_orders_the_kv_reads(kv_fp32):
    """K/V written on another stream behind a long wait: calls given the
    writer's event return exactly what calls on ready K/V return (a call that
    read K/V before the event would see the zero-filled buffers)."""
    wl, routes, q, k, v, do = _inputs("thd16k", 1024)
    out, lse = qsa.forward(q, k, v, routes, wl.scale)
    ref = qsa.backward(do, q, k, v, out, lse, routes, wl.scale, kv_fp32=kv_fp32)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()

    def late_kv():
        kb, vb = torch.zeros_like(k), torch.zeros_like(v)
        side = torch.cuda.Stream()
        side.wait_stream(main)
        with torch.cuda.stream(side):
            torch.cuda._sleep(100_000_000)  # a bounded spin, tens of milliseconds
            kb.copy_(k)
            vb.copy_(v)
            ready = torch.cuda.Event()
            ready.record(side)
        kb.record_stream(main)
        vb.record_stream(main)
        return kb, vb, ready

    kb, vb, ready = late_kv()
    o2, l2 = qsa.forward(q, kb, vb, routes, wl.scale, kv_ready=ready)
    kb, vb, ready = late_kv()
    got = qsa.backward(do, q, kb, vb, out, lse, routes, wl.scale, kv_fp32=kv_fp32, kv_ready=ready)
    torch.cuda.synchronize()
    assert torch.equal(o2, out) and torch.equal(l2, lse)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def _rne_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of FP32 to BF16, as bit patterns: add half an ulp of
    the BF16 result (minus one when the kept part is even, so that exact ties go
    to the even neighbour) and drop the low 16 bits; NaNs are left to the caller."""
    b = x32.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    return ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 31, 4096 + 5, 1 << 20])
def test_cast_f32_to_bf16_is_round_to_nearest_even(n):
    rng = np.random.default_rng(n)
    x = (rng.standard_normal(n) * np.exp2(rng.integers(-140, 120, n))).astype(np.float32)
    if n >= 31:
        specials = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 3.4028235e38, -3.4028235e38],
                            dtype=np.float32)
        x[:8] = specials
        # exact ties: low half exactly 0x8000 above an even and an odd BF16 value
        x[8:12] = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x00018000], dtype=np.uint32).view(np.float32)
        x[12] = np.nan
    xd = torch.from_numpy(x).to(DEV)
    y = qsa.cast_f32_to_bf16(xd)
    torch.cuda.synchronize()
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], _rne_bf16_bits(x)[~nan])
    assert np.all(np.isnan(y.cpu().float().numpy()[nan]))
    assert torch.equal(y[~torch.from_numpy(nan).to(DEV)], xd[~torch.from_numpy(nan).to(DEV)].to(torch.bfloat16))
