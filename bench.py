#!/usr/bin/env python
"""QSA forward + backward benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full pass of the hot path on one sequence of the seq32k workload
(T = 32768 tokens, 24 query heads / 2 KV heads, d = 256, 128 four-token blocks
= 512 unique routed keys per query, 564 route slots with 10% duplicates):
route sort/dedup + forward + route transpose + dQ + dK/dV, every kernel of the
library, inputs resident in HBM.  The backward reuses the forward's sorted route
lists from the forward's workspace (qsa_backward_saved), as a training step
keeps them for its backward.  The metric is selected (query, key) token
pairs per second, N = sum_t |R_t| per step (the two KV groups share the routes).

With N GPUs (torchrun), every rank runs its own sequence (independent problems,
no collective on the data path) and the reported value is the sum over ranks of
pairs / the slowest rank's time (weak scaling).

``--impl reference`` times the FP64 CPU oracle on the host cores (each step a
bounded sample of query rows of the same workload) and prints the same line
with ``"impl": "reference"``.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "seq32k"
METRIC = "QSA fwd+bwd selected pairs/s and TFLOP/s at T=32K, 512 sel/query; % roofline"
UNIT = "pairs/s"
FWD_FLOPS_PER_PAIR_HEAD = 4 * 256      # QK^T + PV
BWD_FLOPS_PER_PAIR_HEAD = 10 * 256     # S recompute, dP, dV, dQ, dK
DKDV_FLOPS_PER_PAIR_HEAD = 4 * 256     # dK = dS^T Q, dV = P^T dO
SPEC_BF16_TFLOPS = 2250.0              # B200 dense BF16 tensor peak (NVIDIA specification)
# DRAM bytes (read + write) per step of a stage's kernel, from the ncu capture
# summarised under profiles/, valid only for the sources it was taken on:
# stage -> (bytes per step, {source file: sha256 of that file at capture time}).
TRAFFIC = {
    # the timed step's dK/dV launch on seq32k: ncu dram__bytes_read.sum + dram__bytes_write.sum
    # (the dK/dV summary under profiles/); the file holds the kernel and the phase sizing of its launch
    "bwd_dkdv": (14818692864, {
        "token_indexed_sparse_b200/csrc/qsa_dkdv_union.cu":
            "c650e98ff4ccfb8ca6e8c7eb14b8b19cdfce9b68cbfa355bd7b39c4da2064cbf",
    }),
}


def stage_traffic(stage):
    import hashlib
    if stage not in TRAFFIC:
        return None
    nbytes, sources = TRAFFIC[stage]
    for rel, digest in sources.items():
        with open(os.path.join(ROOT, rel), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    return nbytes


FWD_STAGES = ["fwd_route_rows", "fwd_attention"]
BWD_STAGES = ["bwd_delta_masks", "bwd_tile_lists", "bwd_tile_worklist", "bwd_dq", "bwd_dkdv"]


def pass_ms(stage_ms):
    """Forward, backward and their sum (ms per step) from the per-stage means."""
    fwd = sum(stage_ms.get(n, 0.0) for n in FWD_STAGES)
    bwd = sum(stage_ms.get(n, 0.0) for n in BWD_STAGES)
    return {"forward": fwd, "backward": bwd, "total": fwd + bwd}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def workload_config(wl):
    return {"workload": f"{wl.name}: T={wl.T}, T_kv={wl.T_kv}, {wl.H}Q/{wl.G}KV, d=256, "
                        f"{wl.blocks} four-token blocks (512 unique keys)/query, {wl.W} route slots "
                        f"with 10% duplicates, scale=1/16",
            "T": wl.T, "T_kv": wl.T_kv, "H": wl.H, "G": wl.G, "n_sel": wl.W, "seed": wl.seed}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_step(wl, routes, tens, rows):
    """One oracle fwd+bwd over the given query rows; returns (seconds, pairs)."""
    import oracle
    q, k, v, do = tens
    t0 = time.perf_counter()
    oracle.forward_rows(q, k, v, routes, wl.scale, rows)
    oracle.backward_rows(do, q, k, v, routes, wl.scale, rows)
    dt = time.perf_counter() - t0
    pairs = sum(len(s) for s in oracle.row_route_sets(routes[rows], wl.T_kv))
    return dt, pairs


def oracle_inputs(wl):
    from token_indexed_sparse_b200 import workloads as W
    routes = W.make_routes(wl)
    q, k, v, do = W.make_tensors(wl)
    f = lambda x: x.float().numpy().astype(np.float64)  # noqa: E731
    return routes, (f(q), f(k), f(v), f(do))


def cpu_baseline(wl, budget_s=15.0, seed=0):
    """Oracle (as it stands) on a bounded random sample of query rows."""
    routes, tens = oracle_inputs(wl)
    rng = np.random.default_rng(seed)
    dt, pairs = oracle_sample_step(wl, routes, tens, np.sort(rng.choice(wl.T, 16, replace=False)))
    n_rows = int(min(wl.T, max(16, 16 * budget_s / max(dt, 1e-3))))
    rows = np.sort(rng.choice(wl.T, n_rows, replace=False))
    dt, pairs = oracle_sample_step(wl, routes, tens, rows)
    return {"value": pairs / dt, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"FP64 row-gather oracle, forward+backward over {n_rows} random query rows "
                      f"({pairs} pairs) of the same workload, {dt:.1f} s"}


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def run_reference(args):
    """The reference arm: the CPU oracle, a bounded row sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from token_indexed_sparse_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]          # the same workload as the CUDA arm
    if args.scale_T:
        wl = wl.scaled(args.scale_T)
    routes, tens = oracle_inputs(wl)
    rng = np.random.default_rng(1)
    rows_per_step = args.reference_rows
    for _ in range(args.warmup):
        oracle_sample_step(wl, routes, tens, np.sort(rng.choice(wl.T, rows_per_step, replace=False)))
    total_t, total_p = 0.0, 0
    for _ in range(args.steps):
        dt, p = oracle_sample_step(wl, routes, tens, np.sort(rng.choice(wl.T, rows_per_step, replace=False)))
        total_t += dt
        total_p += p
    value = total_p / total_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"FP64 row-gather oracle, forward+backward over {rows_per_step} random "
                                       f"query rows per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bitmap_adapter_aux(qsa, torch, routes, wl, dev, flush, peaks, reps=10):
    """Times the bitmap -> route IDs adapter on this workload's routes rendered as
    a single-sequence block bitmap (an auxiliary line: not part of the step)."""
    T, T_kv = wl.T, wl.T_kv
    NB = (T_kv + 3) // 4
    if T * NB > (1 << 32):
        return None
    sel = torch.zeros((T, NB), dtype=torch.uint8, device=dev)
    valid = (routes >= 0) & (routes < T_kv)
    rows = torch.arange(T, device=dev).unsqueeze(1).expand_as(routes)[valid]
    sel[rows, (routes[valid] // 4).long()] = 1
    zero = torch.zeros(T, dtype=torch.int32, device=dev)
    hi = torch.arange(T, dtype=torch.int32, device=dev) + wl.q_offset
    for _ in range(2):
        qsa.bitmap_routes(sel, zero, hi, zero, zero, T_kv, wl.W)
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qsa.bitmap_routes(sel, zero, hi, zero, zero, T_kv, wl.W)
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    t = np.arange(T, dtype=np.int64) + wl.q_offset
    scanned = int(np.minimum(t // 4, NB - 1).sum() + T)      # bitmap bytes in each row's reachable range
    nbytes = scanned + 16 * T + 4 * T * wl.W + 4 * T
    avg = float(np.mean(ms))
    del sel
    return {"kernel": "bitmap_routes", "workload": f"{wl.name} routes as a [{T}, {NB}] uint8 block bitmap",
            "ms": avg, "bytes": nbytes, "bound": "hbm", "achieved": nbytes / (avg * 1e-3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": nbytes / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"]}


def selector_aux(qsa, torch, dev, flush, peaks, T=32768, Hi=64, NB=8192, k=127, reps=5):
    """Times the block selector on the seq32k shape (an auxiliary line: not part of
    the step): tcgen05 scores of every candidate block, then top-k + expansion."""
    g = torch.Generator(device=dev).manual_seed(4321)
    qi = torch.randn(T, Hi, 128, device=dev, generator=g).to(torch.bfloat16)
    kbar = torch.randn(NB, 128, device=dev, generator=g).to(torch.bfloat16)
    scores = torch.empty(T, NB, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):
        qsa.selector_scores(qi, kbar, 1 / 64, scores=scores, status=status)
        qsa.selector_topk(scores, k, NB)
    torch.cuda.synchronize()
    ms_s, ms_k = [], []
    for _ in range(reps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        qsa.selector_scores(qi, kbar, 1 / 64, scores=scores, status=status)
        e[1].record()
        qsa.selector_topk(scores, k, NB)
        e[2].record()
        torch.cuda.synchronize()
        ms_s.append(e[0].elapsed_time(e[1]))
        ms_k.append(e[1].elapsed_time(e[2]))
    n = np.minimum(np.arange(T, dtype=np.int64) // 4, NB)
    flops = 2.0 * Hi * 128 * float(n.sum())
    avg_s, avg_k = float(np.mean(ms_s)), float(np.mean(ms_k))
    ok = int(status.item()) == 0
    del qi, kbar, scores
    return {"kernel": "selector_scores (tcgen05)", "workload": f"T={T}, {Hi} indexer heads x 128 dims, NB={NB} "
            f"compressed blocks, top-{k} + tail", "ms": avg_s, "bound": "tensor", "flops": flops,
            "achieved": flops / (avg_s * 1e-3) / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": flops / (avg_s * 1e-3) / 1e12 / peaks["bf16_tflops"], "topk_ms": avg_k, "status_ok": ok}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from token_indexed_sparse_b200 import qsa
    from token_indexed_sparse_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    wl = W.WORKLOADS[args.workload]
    if args.scale_T:
        wl = wl.scaled(args.scale_T)
    routes_np = np.array(W.make_routes(wl), dtype=np.int32)
    q_h, k_h, v_h, do_h = W.make_tensors(wl)
    pairs = W.pair_count(routes_np, wl.T_kv)
    flops = (FWD_FLOPS_PER_PAIR_HEAD + BWD_FLOPS_PER_PAIR_HEAD) * wl.H * pairs
    routes_h = torch.from_numpy(routes_np)
    host_in = [t.pin_memory() for t in (q_h, k_h, v_h, do_h, routes_h)]
    q, k, v, do, routes = (t.to(dev) for t in host_in)
    out = torch.empty_like(q)
    lse = torch.empty(wl.T, wl.H, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = torch.empty(qsa.forward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, wl.W), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(qsa.backward_workspace_size(wl.T, wl.T_kv, wl.H, wl.G, wl.W), dtype=torch.uint8,
                       device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step(fwd_ev=None, bwd_ev=None):
        qsa.forward(q, k, v, routes, wl.scale, out=out, lse=lse, workspace=ws_f, stage_events=fwd_ev)
        # the backward reuses the forward's route lists (kept in ws_f) instead of sorting again
        qsa.backward(do, q, k, v, out, lse, routes, wl.scale, dq=dq, dk=dk, dv=dv, workspace=ws_b,
                     stage_events=bwd_ev, saved_workspace=ws_f)

    for _ in range(args.warmup):
        step()
        flush.zero_()
    torch.cuda.synchronize()

    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    starts = [mk() for _ in range(args.steps)]
    fwd_ev = [[mk() for _ in FWD_STAGES] for _ in range(args.steps)]
    bwd_ev = [[mk() for _ in BWD_STAGES] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()                 # L2 flushed before every timed step (outside its events)
        starts[i].record(stream)
        step(fwd_ev[i], bwd_ev[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()

    stage_ms = {n: [] for n in FWD_STAGES + BWD_STAGES}
    step_ms = []
    for i in range(args.steps):
        prev = starts[i]
        for n, e in zip(FWD_STAGES + BWD_STAGES, fwd_ev[i] + bwd_ev[i]):
            stage_ms[n].append(prev.elapsed_time(e))
            prev = e
        step_ms.append(starts[i].elapsed_time(bwd_ev[i][-1]))
    total_ms = float(sum(step_ms))
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * pairs * args.steps / (total_ms * 1e-3)

    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"workload": wl.name, "ms_per_step": ms_per_step,
                              "stage_ms": {n: float(np.mean(v)) for n, v in stage_ms.items()}}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # end to end through the public API: pinned host inputs -> device, fwd+bwd, results -> pinned host
    res_h = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (out, lse, dq, dk, dv)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in res_h)

    # Pipelined: step i's inputs go in on s_in while step i-1 computes on the bench
    # stream and step i-2's results come out on s_out (two device buffer sets; the
    # two copy directions use separate copy engines).  Every step's bytes cross the
    # bus inside the timed region.
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    d_in = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in host_in] for _ in range(2)]
    d_res = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in res_h] for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of set b landed
    ev_cmp = [torch.cuda.Event() for _ in range(2)]   # set b computed (its inputs consumed)
    ev_out = [torch.cuda.Event() for _ in range(2)]   # results of set b copied out

    def e2e_run(n_steps):
        for i in range(n_steps + 2):
            if i < n_steps:
                b = i & 1
                if i >= 2:
                    s_in.wait_event(ev_cmp[b])
                with torch.cuda.stream(s_in):
                    for d, h in zip(d_in[b], host_in):
                        d.copy_(h, non_blocking=True)
                ev_in[b].record(s_in)
            j = i - 1
            if 0 <= j < n_steps:
                b = j & 1
                stream.wait_event(ev_in[b])
                if j >= 2:
                    stream.wait_event(ev_out[b])
                q_, k_, v_, do_, r_ = d_in[b]
                o_, l_, dq_, dk_, dv_ = d_res[b]
                qsa.forward(q_, k_, v_, r_, wl.scale, out=o_, lse=l_, workspace=ws_f)
                qsa.backward(do_, q_, k_, v_, o_, l_, r_, wl.scale, dq=dq_, dk=dk_, dv=dv_, workspace=ws_b,
                             saved_workspace=ws_f)
                ev_cmp[b].record(stream)
            kk = i - 2
            if 0 <= kk < n_steps:
                b = kk & 1
                s_out.wait_event(ev_cmp[b])
                with torch.cuda.stream(s_out):
                    for h, d in zip(res_h, d_res[b]):
                        h.copy_(d, non_blocking=True)
                ev_out[b].record(s_out)

    # enough steps that the pipeline's fill (the first inputs) and drain (the
    # last results) weigh little against the steady state (about 1 s of copies)
    e2e_steps = max(40, args.steps)
    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = mk(), mk()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    e2e_run(e2e_steps)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * pairs * e2e_steps / (e2e_ms * 1e-3)
    del d_in, d_res

    peaks = load_peaks()
    avg = {n: float(np.mean(v)) for n, v in stage_ms.items()}
    dominant = max(avg, key=avg.get)
    # algorithmic work of the dominant kernel per launch
    if dominant == "bwd_dkdv":
        work = DKDV_FLOPS_PER_PAIR_HEAD * wl.H * pairs
    elif dominant == "bwd_dq":
        work = (BWD_FLOPS_PER_PAIR_HEAD - DKDV_FLOPS_PER_PAIR_HEAD) * wl.H * pairs
    elif dominant == "fwd_attention":
        work = FWD_FLOPS_PER_PAIR_HEAD * wl.H * pairs
    else:
        work = None
    roofline = None
    if work is not None:
        achieved = work / (avg[dominant] * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": stage_traffic(dominant),
                    "peak_source": f"{peaks['source']} bf16_tflops (burst; the timed region is well under a "
                                   f"second)",
                    "frac_of_spec": achieved / SPEC_BF16_TFLOPS}
    aux = {"bitmap_routes": bitmap_adapter_aux(qsa, torch, routes, wl, dev, flush, peaks),
           "selector": selector_aux(qsa, torch, dev, flush, peaks)}
    step_tflops = flops / (ms_per_step * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(wl), "pairs_per_step": pairs, "flops_per_step": flops,
                   "l2": "flushed (256 MiB write) before every timed step, outside its events",
                   "backward": "on the forward's saved route lists (qsa_backward_saved)",
                   "parallelism": f"{world} independent sequences (one per GPU)" if world > 1 else "1 GPU"},
        "tflops": step_tflops * world,
        "step_roofline": {"flops": flops, "t_roof_ms": flops / (peaks["bf16_tflops"] * 1e12) * 1e3,
                          "frac": step_tflops / peaks["bf16_tflops"],
                          "peak": peaks["bf16_tflops"], "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                          "frac_of_spec": step_tflops / SPEC_BF16_TFLOPS},
        "stage_ms": avg,
        "pass_ms": pass_ms(avg),
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                "how": "pinned host -> device inputs, forward + backward through the C ABI, device -> pinned host "
                       "results, every step; copies of neighbouring steps overlap the kernels on two copy streams"},
        "gpu_launches": args.steps * (qsa.launch_count(wl.T, wl.T_kv, wl.H, wl.G, wl.W, False)
                                      + qsa.launch_count(wl.T, wl.T_kv, wl.H, wl.G, wl.W, True)),
        "clocks": clk,
        "aux": aux,
    }
    if world > 1:
        dist.barrier()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_cp(args):
    """Context parallelism: ONE sequence of the workload (cp128k by default: 8192
    query rows against 131072 K/V rows) split across the ranks through
    token_indexed_sparse_b200.cp: each rank owns a pair-balanced range of query
    rows and an equal slice of K/V; a step is the CP forward (K/V all-gather,
    local forward) and the CP backward (all-gather, local FP32 dK/dV backward,
    FP32 reduce-scatter, BF16 rounding of the own slice), collectives inside the
    timed region.  Total work is fixed as the rank count grows (strong scaling)."""
    import datetime

    import torch
    import torch.distributed as dist

    from token_indexed_sparse_b200 import cp, qsa
    from token_indexed_sparse_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    else:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                device_id=dev, timeout=datetime.timedelta(seconds=120))
    wl = W.WORKLOADS[args.workload if args.workload != WORKLOAD else "cp128k"]
    if args.scale_T:
        wl = wl.scaled(args.scale_T)
    routes_np = np.array(W.make_routes(wl), dtype=np.int32)
    counts = np.array([np.unique(r[(r >= 0) & (r < wl.T_kv)]).size for r in routes_np])
    s, e = cp.balanced_query_ranges(counts, world)[rank]
    ks, ke = cp.kv_slice(wl.T_kv, world, rank)
    q_h, k_h, v_h, do_h = W.make_tensors(wl)
    pairs_total = int(counts.sum())
    host_in = [t.contiguous().pin_memory() for t in (q_h[s:e], k_h[ks:ke], v_h[ks:ke], do_h[s:e],
                                                     torch.from_numpy(routes_np[s:e]))]
    q, k, v, do, routes = (t.to(dev) for t in host_in)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    ws_f = torch.empty(qsa.forward_workspace_size(e - s, wl.T_kv, wl.H, wl.G, wl.W), dtype=torch.uint8, device=dev)

    def step(q_, k_, v_, do_, r_):
        out, lse = cp.cp_forward(q_, k_, v_, r_, wl.scale, workspace=ws_f)
        return (out, lse, *cp.cp_backward(do_, q_, k_, v_, out, lse, r_, wl.scale, saved_workspace=ws_f))

    for _ in range(args.warmup):
        step(q, k, v, do, routes)
        flush.zero_()
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [(mk(), mk()) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()                 # L2 flushed before every timed step (outside its events)
        ev[i][0].record(stream)
        step(q, k, v, do, routes)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    t = torch.tensor([sum(a.elapsed_time(b) for a, b in ev)], device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    value = pairs_total * args.steps / (total_ms * 1e-3)

    # end to end: this rank's inputs in from pinned host memory, the CP step,
    # its results (out, lse, dq, own dk / dv slices) back to pinned host memory
    res_shapes = [(e - s, wl.H, 256), (e - s, wl.H), (e - s, wl.H, 256), (ke - ks, wl.G, 256), (ke - ks, wl.G, 256)]
    res_types = [torch.bfloat16, torch.float32, torch.bfloat16, torch.bfloat16, torch.bfloat16]
    res_h = [torch.empty(sh, dtype=ty, pin_memory=True) for sh, ty in zip(res_shapes, res_types)]
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = sum(x.numel() * x.element_size() for x in res_h)
    e2e_steps = max(3, args.steps // 2)
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = mk(), mk()
    e0.record(stream)
    for _ in range(e2e_steps):
        ins = [x.to(dev, non_blocking=True) for x in host_in]
        for dst, src in zip(res_h, step(*ins)):
            dst.copy_(src, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_value = pairs_total * e2e_steps / (float(t.item()) * 1e-3)
    flops = (FWD_FLOPS_PER_PAIR_HEAD + BWD_FLOPS_PER_PAIR_HEAD) * wl.H * pairs_total
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(wl), "pairs_per_step": pairs_total, "flops_per_step": flops,
                   "l2": "flushed (256 MiB write) before every timed step, outside its events",
                   "backward": "on the forward's saved route lists (qsa_backward_saved)",
                   "parallelism": f"cp{world}: one sequence, query rows balanced by routed pairs, K/V "
                                  f"all-gather and FP32 dK/dV reduce-scatter over NCCL"},
        "tflops": flops * args.steps / (total_ms * 1e-3) / 1e12,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "how": "per rank: its inputs in, the CP step, its results out, serially"},
        "gpu_launches": args.steps * (qsa.launch_count(e - s, wl.T_kv, wl.H, wl.G, wl.W, False)
                                      + qsa.launch_count(e - s, wl.T_kv, wl.H, wl.G, wl.W, True) + 2),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="time the device-resident steps only and print the stage breakdown (profiling runs)")
    ap.add_argument("--workload", default=WORKLOAD, choices=["tiny", "seq4k", "thd16k", "seq32k", "cp128k"])
    ap.add_argument("--scale-T", type=int, default=0,
                    help="run the workload's recipe at this many query rows (profiling of smaller cases)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--reference-rows", type=int, default=96)
    ap.add_argument("--mode", choices=["replicas", "cp"], default="replicas",
                    help="replicas: one independent sequence per GPU (default); cp: one sequence split across "
                         "the GPUs by context parallelism")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "cp":
        run_cp(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
