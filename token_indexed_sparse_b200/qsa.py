"""Thin Python binding of libqsa_b200.so (argument marshalling only).

Every step of the computation runs in the CUDA library; this module passes
device pointers of PyTorch tensors and the current CUDA stream through the C ABI
declared in ``include/qsa.h``.  There is no fallback: if the library is missing
or the tensors are not on a CUDA device, the call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqsa_b200.so")
_lib = None

QSA_OK = 0


class QSAError(RuntimeError):
    """A QSA C-ABI call returned a non-OK status."""

    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {status_string(status)} ({status})")
        self.status = status


def library() -> ctypes.CDLL:
    """Load the shared library (once); raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"QSA CUDA library not found at {_LIB_PATH}; build it with "
            "`python -m token_indexed_sparse_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.qsa_status_string.restype = ctypes.c_char_p
    lib.qsa_status_string.argtypes = [i32]
    lib.qsa_version.restype = ctypes.c_char_p
    lib.qsa_version.argtypes = []
    for name in ("qsa_forward_workspace_size", "qsa_backward_workspace_size"):
        f = getattr(lib, name)
        f.restype = sz
        f.argtypes = [i64, i64, i32, i32, i32]
    lib.qsa_forward.restype = i32
    lib.qsa_forward.argtypes = [vp, vp, vp, vp, i64, i64, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    lib.qsa_backward.restype = i32
    lib.qsa_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, f32,
                                 vp, vp, vp, vp, sz, vp]
    lib.qsa_forward_ex.restype = i32
    lib.qsa_forward_ex.argtypes = lib.qsa_forward.argtypes + [vp, i32]
    lib.qsa_backward_ex.restype = i32
    lib.qsa_backward_ex.argtypes = lib.qsa_backward.argtypes + [vp, i32]
    lib.qsa_forward_kvwait.restype = i32
    lib.qsa_forward_kvwait.argtypes = lib.qsa_forward.argtypes + [vp, vp, i32]
    lib.qsa_backward_saved.restype = i32
    lib.qsa_backward_saved.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i64, i64, i32, i32, i32, f32, vp, vp, vp, i32,
                                       vp, sz, vp, vp, vp, i32]
    lib.qsa_backward_kvwait.restype = i32
    lib.qsa_backward_kvwait.argtypes = lib.qsa_backward.argtypes[:16] + [i32] + lib.qsa_backward.argtypes[16:] + [
        vp, vp, i32]
    lib.qsa_launch_count.restype = i32
    lib.qsa_launch_count.argtypes = [i64, i64, i32, i32, i32, i32]
    lib.qsa_bitmap_routes.restype = i32
    lib.qsa_bitmap_routes.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp]
    lib.qsa_selector_scores.restype = i32
    lib.qsa_selector_scores.argtypes = [vp, vp, i64, i64, i32, i32, f32, vp, vp, vp, vp, i64, vp, vp]
    lib.qsa_selector_topk.restype = i32
    lib.qsa_selector_topk.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp]
    lib.qsa_backward_fp32kv.restype = i32
    lib.qsa_backward_fp32kv.argtypes = lib.qsa_backward.argtypes
    lib.qsa_route_plan_scratch_size.restype = sz
    lib.qsa_route_plan_scratch_size.argtypes = [i64, i64]
    lib.qsa_route_plan.restype = i32
    lib.qsa_route_plan.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.qsa_tile_plan_scratch_size.restype = sz
    lib.qsa_tile_plan_scratch_size.argtypes = [i64, i64]
    lib.qsa_tile_plan.restype = i32
    lib.qsa_tile_plan.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.qsa_union_group.restype = i32
    lib.qsa_union_group.argtypes = [i32]
    lib.qsa_union_plan.restype = i32
    lib.qsa_union_plan.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp, vp, vp]
    lib.qsa_cast_f32_to_bf16.restype = i32
    lib.qsa_cast_f32_to_bf16.argtypes = [vp, vp, i64, vp]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return library().qsa_status_string(int(status)).decode()


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status: int, what: str):
    if status != QSA_OK:
        raise QSAError(status, what)


def _prep(x: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {x.dtype}")
    return x.contiguous()


def _out(t: torch.Tensor, shape, dtype, device, name: str) -> torch.Tensor:
    """A caller-provided output buffer.  The kernels write it in place through its
    pointer, so it must be exactly the dense tensor they expect: anything else
    is refused before the call (a strided or short buffer would be overrun)."""
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _sizes(q, k, routes):
    if q.dim() != 3 or k.dim() != 3 or routes.dim() != 2:
        raise ValueError("expected q [T,H,256], k/v [T_kv,G,256], routes [T,n_sel]")
    T, H, D = q.shape
    T_kv, G, Dk = k.shape
    if D != 256 or Dk != 256:
        raise ValueError("head dimension must be 256")
    if routes.shape[0] != T:
        raise ValueError("routes must have one row per query")
    return T, T_kv, H, G, routes.shape[1]


def forward_workspace_size(T, T_kv, H, G, n_sel) -> int:
    return int(library().qsa_forward_workspace_size(T, T_kv, H, G, n_sel))


def backward_workspace_size(T, T_kv, H, G, n_sel) -> int:
    return int(library().qsa_backward_workspace_size(T, T_kv, H, G, n_sel))


def launch_count(T, T_kv, H, G, n_sel, backward: bool) -> int:
    """Kernels one forward / backward call enqueues (0 for rejected sizes)."""
    return int(library().qsa_launch_count(T, T_kv, H, G, n_sel, 1 if backward else 0))


def _workspace(nbytes: int, device, given: torch.Tensor | None) -> torch.Tensor:
    if given is not None:  # a dense uint8 buffer: its element count is its size in bytes
        if given.device != device or given.dtype != torch.uint8 or not given.is_contiguous():
            raise ValueError(f"workspace must be a contiguous uint8 tensor on {device}")
        return given
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _events(stage_events):
    """ctypes array of raw cudaEvent_t handles from torch.cuda.Event objects."""
    if not stage_events:
        return None, 0
    handles = []
    for e in stage_events:
        if e.cuda_event == 0:          # torch creates events lazily
            e.record()
        handles.append(e.cuda_event)
    return (ctypes.c_void_p * len(handles))(*handles), len(handles)


def _event_handle(e):
    """Raw cudaEvent_t of a recorded torch.cuda.Event, or None."""
    if e is None:
        return None
    if e.cuda_event == 0:
        raise ValueError("kv_ready must be a recorded torch.cuda.Event")
    return e.cuda_event


def forward(q, k, v, routes, scale: float = 1.0 / 16.0, *, out=None, lse=None, workspace=None,
            stage_events=None, kv_ready=None):
    """qsa_forward: returns ``(out [T,H,256] bf16, lse [T,H] float32)``.

    ``stage_events`` (optional list of torch.cuda.Event) are recorded after the
    route-sort and attention stages.  ``kv_ready`` (optional recorded
    torch.cuda.Event): k and v may still be being written until it fires; the
    route work runs first and the attention waits for it (qsa_forward_kvwait)."""
    lib = library()
    q = _prep(q, torch.bfloat16, "q")
    k = _prep(k, torch.bfloat16, "k")
    v = _prep(v, torch.bfloat16, "v")
    routes = _prep(routes, torch.int32, "routes")
    T, T_kv, H, G, n_sel = _sizes(q, k, routes)
    out = torch.empty_like(q) if out is None else _out(out, q.shape, torch.bfloat16, q.device, "out")
    lse = (torch.empty(T, H, dtype=torch.float32, device=q.device) if lse is None
           else _out(lse, (T, H), torch.float32, q.device, "lse"))
    ws_bytes = lib.qsa_forward_workspace_size(T, T_kv, H, G, n_sel)
    ws = _workspace(ws_bytes, q.device, workspace)
    ev, n_ev = _events(stage_events)
    st = lib.qsa_forward_kvwait(_ptr(q), _ptr(k), _ptr(v), _ptr(routes), T, T_kv, H, G, n_sel, float(scale),
                                _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device),
                                _event_handle(kv_ready), ev, n_ev)
    _check(st, "qsa_forward")
    return out, lse


def backward(grad_out, q, k, v, out, lse, routes, scale: float = 1.0 / 16.0, *,
             dq=None, dk=None, dv=None, workspace=None, stage_events=None, kv_fp32: bool = False,
             kv_ready=None, saved_workspace=None):
    """qsa_backward: returns ``(dq, dk, dv)`` (bf16, shapes of q, k, v).

    ``stage_events`` (optional, up to 5 torch.cuda.Event) are recorded after
    each backward stage.  With ``kv_fp32`` dk and dv are FP32 (the sums before
    the BF16 rounding, for adding partials from several calls).  ``kv_ready``
    (optional recorded torch.cuda.Event): k and v may still be being written
    until it fires; the route work runs first and dQ waits for it
    (qsa_backward_kvwait).  ``saved_workspace``: the workspace tensor of the
    forward call on the same routes (still holding its route lists, which
    are then reused instead of sorting the routes again: qsa_backward_saved);
    ``routes`` then only gives n_sel."""
    lib = library()
    grad_out = _prep(grad_out, torch.bfloat16, "grad_out")
    q = _prep(q, torch.bfloat16, "q")
    k = _prep(k, torch.bfloat16, "k")
    v = _prep(v, torch.bfloat16, "v")
    out = _prep(out, torch.bfloat16, "out")
    lse = _prep(lse, torch.float32, "lse")
    routes = _prep(routes, torch.int32, "routes")
    T, T_kv, H, G, n_sel = _sizes(q, k, routes)
    kv_dtype = torch.float32 if kv_fp32 else torch.bfloat16
    dq = torch.empty_like(q) if dq is None else _out(dq, q.shape, torch.bfloat16, q.device, "dq")
    dk = (torch.empty(k.shape, dtype=kv_dtype, device=k.device) if dk is None
          else _out(dk, k.shape, kv_dtype, k.device, "dk"))
    dv = (torch.empty(v.shape, dtype=kv_dtype, device=v.device) if dv is None
          else _out(dv, v.shape, kv_dtype, v.device, "dv"))
    ws_bytes = lib.qsa_backward_workspace_size(T, T_kv, H, G, n_sel)
    ws = _workspace(ws_bytes, q.device, workspace)
    ev, n_ev = _events(stage_events)
    if saved_workspace is not None:
        fws = _workspace(0, q.device, saved_workspace)
        st = lib.qsa_backward_saved(_ptr(grad_out), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(fws),
                                    fws.numel(), T, T_kv, H, G, n_sel, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                                    1 if kv_fp32 else 0, _ptr(ws), ws.numel(), _stream(q.device),
                                    _event_handle(kv_ready), ev, n_ev)
        _check(st, "qsa_backward_saved")
        return dq, dk, dv
    st = lib.qsa_backward_kvwait(_ptr(grad_out), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(routes),
                                 T, T_kv, H, G, n_sel, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                                 1 if kv_fp32 else 0, _ptr(ws), ws.numel(), _stream(q.device),
                                 _event_handle(kv_ready), ev, n_ev)
    _check(st, "qsa_backward")
    return dq, dk, dv


def union_plan(routes, T_kv: int):
    """qsa_union_plan: ``(group, ucnt, ukey, uown)`` of the forward's query
    groups (route rows first, as qsa_route_plan); ``ukey`` / ``uown`` are
    ``[n_groups, group * n_sel]``, row i valid up to ``ucnt[i]``."""
    lib = library()
    routes = _prep(routes, torch.int32, "routes")
    T, n_sel = routes.shape
    group = lib.qsa_union_group(n_sel)
    if group < 1:
        raise ValueError("n_sel outside 1..16384")
    n_groups = (T + group - 1) // group
    dev = routes.device
    row_cnt = torch.empty(T, dtype=torch.int32, device=dev)
    row_cols = torch.empty(T, n_sel, dtype=torch.int32, device=dev)
    ucnt = torch.empty(n_groups, dtype=torch.int32, device=dev)
    ukey = torch.empty(n_groups, group * n_sel, dtype=torch.int32, device=dev)
    uown = torch.empty(n_groups, group * n_sel, dtype=torch.uint8, device=dev)
    _check(lib.qsa_union_plan(_ptr(routes), T, T_kv, n_sel, _ptr(row_cnt), _ptr(row_cols), _ptr(ucnt), _ptr(ukey),
                              _ptr(uown), _stream(dev)), "qsa_union_plan")
    return group, ucnt, ukey, uown


def cast_f32_to_bf16(x, out=None):
    """qsa_cast_f32_to_bf16: ``x`` (FP32, CUDA) rounded to BF16, to nearest even.

    The final rounding of FP32 dK/dV sums added up across calls (context
    parallelism), the same rounding the backward applies itself."""
    lib = library()
    x = _prep(x, torch.float32, "x")
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else \
        _out(out, x.shape, torch.bfloat16, x.device, "out")
    if x.data_ptr() % 16 or out.data_ptr() % 16:
        raise ValueError("x and out must be 16-byte aligned")
    _check(lib.qsa_cast_f32_to_bf16(_ptr(x), _ptr(out), x.numel(), _stream(x.device)), "qsa_cast_f32_to_bf16")
    return out


def route_plan(routes, T_kv: int):
    """qsa_route_plan: ``(row_cnt, row_cols, quad_ptr, quad_ent)`` device tensors."""
    lib = library()
    routes = _prep(routes, torch.int32, "routes")
    T, n_sel = routes.shape
    dev = routes.device
    nq = (T_kv + 3) // 4
    row_cnt = torch.empty(T, dtype=torch.int32, device=dev)
    row_cols = torch.empty(T, n_sel, dtype=torch.int32, device=dev)
    quad_ptr = torch.empty(nq + 1, dtype=torch.int32, device=dev)
    quad_ent = torch.empty(T * n_sel, dtype=torch.int64, device=dev)
    scratch = torch.empty(max(256, lib.qsa_route_plan_scratch_size(T, T_kv)), dtype=torch.uint8, device=dev)
    st = lib.qsa_route_plan(_ptr(routes), T, T_kv, n_sel, _ptr(row_cnt), _ptr(row_cols), _ptr(quad_ptr),
                            _ptr(quad_ent), _ptr(scratch), scratch.numel(), _stream(dev))
    _check(st, "qsa_route_plan")
    return row_cnt, row_cols, quad_ptr, quad_ent


def tile_plan(routes, T_kv: int):
    """qsa_tile_plan: ``(row_cnt, row_cols, tile_ptr, tile_ent)`` device tensors."""
    lib = library()
    routes = _prep(routes, torch.int32, "routes")
    T, n_sel = routes.shape
    dev = routes.device
    nt = (T_kv + 127) // 128
    row_cnt = torch.empty(T, dtype=torch.int32, device=dev)
    row_cols = torch.empty(T, n_sel, dtype=torch.int32, device=dev)
    tile_ptr = torch.empty(nt + 1, dtype=torch.int32, device=dev)
    tile_ent = torch.empty(T * n_sel, dtype=torch.int64, device=dev)
    scratch = torch.empty(max(256, lib.qsa_tile_plan_scratch_size(T, T_kv)), dtype=torch.uint8, device=dev)
    st = lib.qsa_tile_plan(_ptr(routes), T, T_kv, n_sel, _ptr(row_cnt), _ptr(row_cols), _ptr(tile_ptr),
                           _ptr(tile_ent), _ptr(scratch), scratch.numel(), _stream(dev))
    _check(st, "qsa_tile_plan")
    return row_cnt, row_cols, tile_ptr, tile_ent


def bitmap_routes(sel_blocks, lo, hi, blk_base, tok_base, T_kv: int, n_sel: int, block_size: int = 4):
    """Bitmap selection -> route IDs on the GPU (``qsa_bitmap_routes``).

    Returns ``(routes [T, n_sel] int32, row_cnt [T] int32, max_cnt [1] int32)``,
    all on the device and produced asynchronously on the current stream.
    """
    lib = library()
    sel = _prep(sel_blocks, torch.uint8, "sel_blocks")
    dev = sel.device
    T, NB = sel.shape
    lo, hi, blk_base, tok_base = (_prep(x, torch.int32, n) for x, n in
                                  ((lo, "lo"), (hi, "hi"), (blk_base, "blk_base"), (tok_base, "tok_base")))
    routes = torch.empty((T, n_sel), dtype=torch.int32, device=dev)
    row_cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    max_cnt = torch.empty((1,), dtype=torch.int32, device=dev)
    st = lib.qsa_bitmap_routes(_ptr(sel), _ptr(lo), _ptr(hi), _ptr(blk_base), _ptr(tok_base), T, NB, T_kv,
                               block_size, n_sel, _ptr(routes), _ptr(row_cnt), _ptr(max_cnt), _stream(dev))
    _check(st, "qsa_bitmap_routes")
    return routes, row_cnt, max_cnt


def _opt_i32(x, name):
    return None if x is None else _prep(x, torch.int32, name)


def selector_scores(qi, kbar, scale: float, pos=None, blk_base=None, tok_base=None, scores=None, status=None):
    """Candidate block scores on the tensor cores (``qsa_selector_scores``).

    ``qi`` [T, Hi, 128] and ``kbar`` [NB, 128] BF16 on the GPU.  Returns
    ``scores`` [T, NB] FP32 (entries that are not candidates are left as they
    were: NaN in a fresh tensor) and a one-element device status tensor.
    """
    lib = library()
    qi = _prep(qi, torch.bfloat16, "qi")
    kbar = _prep(kbar, torch.bfloat16, "kbar")
    T, Hi, Di = qi.shape
    NB = kbar.shape[0]
    dev = qi.device
    pos, blk_base, tok_base = (_opt_i32(x, n) for x, n in ((pos, "pos"), (blk_base, "blk_base"),
                                                           (tok_base, "tok_base")))
    if scores is None:
        scores = torch.full((T, NB), float("nan"), dtype=torch.float32, device=dev)
    elif (scores.device != dev or scores.dtype != torch.float32 or scores.dim() != 2 or scores.shape[0] != T
          or scores.shape[1] < NB or scores.stride(1) != 1):
        raise ValueError(f"scores must be a float32 [{T}, >= {NB}] tensor on {dev} with unit column stride")
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    elif status.device != dev or status.dtype != torch.int32 or status.numel() < 1 or not status.is_contiguous():
        raise ValueError(f"status must be a contiguous int32 tensor on {dev}")
    st = lib.qsa_selector_scores(_ptr(qi), _ptr(kbar), T, NB, Hi, Di, scale, _ptr(pos), _ptr(blk_base),
                                 _ptr(tok_base), _ptr(scores), scores.stride(0), _ptr(status), _stream(dev))
    _check(st, "qsa_selector_scores")
    return scores, status


def selector_topk(scores, k: int, NB: int, pos=None, blk_base=None, tok_base=None):
    """Top-k local blocks and expanded token routes (``qsa_selector_topk``)."""
    lib = library()
    scores = _prep(scores, torch.float32, "scores")
    T = scores.shape[0]
    dev = scores.device
    pos, blk_base, tok_base = (_opt_i32(x, n) for x, n in ((pos, "pos"), (blk_base, "blk_base"),
                                                           (tok_base, "tok_base")))
    blocks = torch.empty((T, k), dtype=torch.int32, device=dev)
    routes = torch.empty((T, 4 * (k + 1)), dtype=torch.int32, device=dev)
    st = lib.qsa_selector_topk(_ptr(scores), scores.stride(0), T, NB, k, _ptr(pos), _ptr(blk_base), _ptr(tok_base),
                               _ptr(blocks), _ptr(routes), _stream(dev))
    _check(st, "qsa_selector_topk")
    return blocks, routes


def select(qi, kbar, scale: float, k: int, pos=None, blk_base=None, tok_base=None):
    """The whole selector: (scores, blocks, routes, status)."""
    scores, status = selector_scores(qi, kbar, scale, pos, blk_base, tok_base)
    blocks, routes = selector_topk(scores, k, kbar.shape[0], pos, blk_base, tok_base)
    return scores, blocks, routes, status

